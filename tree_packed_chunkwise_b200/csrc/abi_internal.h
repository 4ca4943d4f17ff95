// Internals shared by the translation units of the C ABI: error reporting, launch accounting.
#pragma once
#include <cuda_runtime.h>

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
