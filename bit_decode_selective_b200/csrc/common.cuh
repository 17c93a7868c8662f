// common.cuh -- host-side error plumbing and small device helpers shared by the
// CUDA translation units of the library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <utility>

#include "../../include/sf.h"

namespace sf {

// ---- host: thread-local error message -------------------------------------

void set_error(const char* fmt, ...);
void clear_error();

#define SF_REQUIRE(cond, ...)                  \
  do {                                         \
    if (!(cond)) {                             \
      ::sf::set_error(__VA_ARGS__);            \
      return SF_ERR_INVALID_ARG;               \
    }                                          \
  } while (0)

#define SF_UNSUPPORTED(cond, ...)              \
  do {                                         \
    if (!(cond)) {                             \
      ::sf::set_error(__VA_ARGS__);            \
      return SF_ERR_UNSUPPORTED;               \
    }                                          \
  } while (0)

// Check the last launch (or a runtime call) and turn a failure into SF_ERR_CUDA.
// The runtime's record of a non-sticky error (a launch refused for its
// resources, say) is cleared, so that it is not reported again by a later,
// unrelated call.
#define SF_CUDA(call)                                                           \
  do {                                                                          \
    cudaError_t e_ = (call);                                                    \
    if (e_ != cudaSuccess) {                                                    \
      (void)cudaGetLastError();                                                 \
      ::sf::set_error("%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_),   \
                      __FILE__, __LINE__);                                      \
      return SF_ERR_CUDA;                                                       \
    }                                                                           \
  } while (0)

#define SF_LAUNCHED() SF_CUDA(cudaGetLastError())

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(sf_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

int num_sms();  // multiprocessors of the current device (cached per device)

// Room left on every SM for the small CTAs of the staging kernels (channel
// selection, row gather), which run on other streams: the kernels that take a
// whole SM per CTA (the refined GEMV, the KV base pass) keep their registers to
// kSideRegs fewer than the SM's 65,536 and their shared memory a block's
// reservation below the SM's, and a staging CTA fits in what is left (at most
// kSideRegs registers, no shared memory), so staging never delays them.
constexpr int kSideRegs = 4096;

// Host-side validation of the descriptor structs (pack.cu).
sf_status check_kv(const sf_kv* kv);
sf_status check_wq_public(const sf_wq* w, bool need_refine);

// ---- device helpers ---------------------------------------------------------

__device__ __forceinline__ double h2d(uint16_t h) {
  return (double)__half2float(__ushort_as_half(h));
}

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Rotary embedding, rotate-half pairing: element i (< d/2) and i + d/2 of a
// head turn by the angle pos * theta^(-2i/d), computed in fp64 so that long
// positions keep their precision; the rotation itself is fp32, each product
// and sum rounded once.
__device__ __forceinline__ void rope_cos_sin(int pos, double theta, int i, int d, float& c, float& s) {
  const double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)d);
  double sn, cs;
  sincos(ang, &sn, &cs);
  c = (float)cs, s = (float)sn;
}
// first (x0 = element i) and second (x1 = element i + d/2) rotated element
__device__ __forceinline__ float rope_first(float x0, float x1, float c, float s) {
  return __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
}
__device__ __forceinline__ float rope_second(float x0, float x1, float c, float s) {
  return __fadd_rn(__fmul_rn(x0, s), __fmul_rn(x1, c));
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now / wait until the previous kernel's results are visible.  Both
// are no-ops when the launch carried no programmatic-serialization attribute.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream is still running.  Every kernel of
// the library starts with pdl_trigger() and calls pdl_wait() before it reads
// anything an earlier kernel wrote, so the chain stays ordered transitively.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace sf
