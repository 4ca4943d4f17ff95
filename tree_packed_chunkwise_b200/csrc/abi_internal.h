// Internals shared by the translation units of the C ABI: error reporting, launch accounting.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdio>
#include <string>
#include <vector>

#include "../../include/tpc.h"
#include "plan.h"

struct tpc_plan {
  tpc::Plan p;
};

namespace tpc_abi {

// records msg as the thread's last error and returns code
int fail(int code, const std::string& msg);

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

template <class KernelT>
cudaError_t set_smem(KernelT k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Index and bounds mode (TPC_CHECKS=1 or tpc_checks_enable): every index field of the plan's
// device tables is bounded on the device before a call that reads them launches anything; returns
// TPC_OK when the mode is off or the tables pass, else TPC_ERR_DEVICE_CHECK (nothing launched).
bool checks_on();
int plan_checks(const tpc_plan* plan, cudaStream_t st);
// the same check of a copy of the plan's tables at `dev` (layout offsets `off`), whatever the mode
int table_checks_at(const tpc::Plan& p, const void* dev, const std::vector<size_t>& off, cudaStream_t st);

// NVTX range over a scope (calls and rounds show up on an Nsight Systems timeline; a few
// nanoseconds when no tool is attached)
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  NvtxRange(const char* name, int round) {
    char buf[48];
    snprintf(buf, sizeof(buf), "%s round %d", name, round);
    nvtxRangePushA(buf);
  }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// multiprocessors of the current device (persistent grids)
int sm_count();
// 2-D bf16 TMA tensor map over [rows][cols] (leading dimension ld_elems): boxes of 64 columns x
// box_rows rows, each box row one 128-byte swizzled line.
bool tensor_map(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t ld_elems, uint32_t box_rows);
// 3-D bf16 TMA tensor map over a [rows][heads][features] tensor: boxes of 64 features x 1 head x
// box_rows rows in the 128-byte-swizzled layout; rows past the end read as zeros.
bool tensor_map_rows(CUtensorMap* m, const void* ptr, uint64_t features, uint64_t heads, uint64_t rows,
                     uint32_t box_rows);

// Optional per-kernel timing: CUDA events around every launch (on the launching stream).
struct Profiler {
  bool on = false;
  long long launches = 0;
  struct Rec { const char* name; cudaEvent_t a, b; };
  std::vector<Rec> recs;
};
extern Profiler g_prof;

}  // namespace tpc_abi

#define TPC_CUDA(call)                                                                  \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess) return tpc_abi::fail(TPC_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

#define TPC_LAUNCH(NAME, STREAM, ...)                                     \
  do {                                                                    \
    cudaEvent_t a_ = nullptr, b_ = nullptr;                               \
    if (tpc_abi::g_prof.on) {                                             \
      TPC_CUDA(cudaEventCreate(&a_));                                     \
      TPC_CUDA(cudaEventCreate(&b_));                                     \
      TPC_CUDA(cudaEventRecord(a_, STREAM));                              \
    }                                                                     \
    __VA_ARGS__;                                                          \
    TPC_CUDA(cudaGetLastError());                                         \
    ++tpc_abi::g_prof.launches;                                           \
    if (tpc_abi::g_prof.on) {                                             \
      TPC_CUDA(cudaEventRecord(b_, STREAM));                              \
      tpc_abi::g_prof.recs.push_back({NAME, a_, b_});                     \
    }                                                                     \
  } while (0)
