// decoder.cu -- the small fp32 kernels that glue the refined projections and
// the refined attention into a Llama-style decoder step: residual add +
// RMSNorm, rotary embedding of q/k, SiLU-gated product, fp32 -> fp16 cast and
// the fp16 LM-head GEMV.  Standard decoder math (the StrataFlux pages run
// their method inside llama.cpp on Llama-3.1-8B and leave these steps as
// they are).
#include <cfloat>

#include "common.cuh"

namespace sf {
namespace {

__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  v = lane < nw ? red[lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  return v;
}

// h[b] += add0[b] + add1[b] (either nullable); x[b] = fp16(h[b] / rms(h[b])).
__global__ void __launch_bounds__(1024) rmsnorm_residual_kernel(float* __restrict__ h,
                                                                const float* __restrict__ add0,
                                                                const float* __restrict__ add1,
                                                                int n, float eps,
                                                                uint16_t* __restrict__ x) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const long row = blockIdx.x;
  float* hr = h + row * n;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    float v = hr[i];
    if (add0) v += add0[row * n + i];
    if (add1) v += add1[row * n + i];
    hr[i] = v;
    ss = fmaf(v, v, ss);
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)n + eps);
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    x[row * n + i] = __half_as_ushort(__float2half_rn(hr[i] * inv));
}

// The same with the row held in registers: thread t owns float4 vectors t,
// t + 1024, ... (VPT of them), all loads of h and the addends issued at once,
// so the row costs one memory round trip and one block reduction.
template <int VPT>
__global__ void __launch_bounds__(1024) rmsnorm_residual_vec_kernel(float* __restrict__ h,
                                                                    const float* __restrict__ add0,
                                                                    const float* __restrict__ add1,
                                                                    int n, float eps,
                                                                    uint16_t* __restrict__ x) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const long row = blockIdx.x;
  const int nv = n / 4;
  float4* h4 = reinterpret_cast<float4*>(h + row * n);
  const float4* a4 = add0 ? reinterpret_cast<const float4*>(add0 + row * n) : nullptr;
  const float4* b4 = add1 ? reinterpret_cast<const float4*>(add1 + row * n) : nullptr;
  float4 v[VPT], a[VPT], c[VPT];
#pragma unroll
  for (int k = 0; k < VPT; k++) {
    const int i = threadIdx.x + 1024 * k;
    const bool in = i < nv;
    v[k] = in ? h4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    a[k] = in && a4 ? a4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    c[k] = in && b4 ? b4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < VPT; k++) {
    const int i = threadIdx.x + 1024 * k;
    v[k].x += a[k].x, v[k].y += a[k].y, v[k].z += a[k].z, v[k].w += a[k].w;
    v[k].x += c[k].x, v[k].y += c[k].y, v[k].z += c[k].z, v[k].w += c[k].w;
    if (i < nv) h4[i] = v[k];
    ss = fmaf(v[k].x, v[k].x, ss);
    ss = fmaf(v[k].y, v[k].y, ss);
    ss = fmaf(v[k].z, v[k].z, ss);
    ss = fmaf(v[k].w, v[k].w, ss);
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)n + eps);
#pragma unroll
  for (int k = 0; k < VPT; k++) {
    const int i = threadIdx.x + 1024 * k;
    if (i < nv) {
      const uint32_t lo = (uint32_t)__half_as_ushort(__float2half_rn(v[k].x * inv)) |
                          ((uint32_t)__half_as_ushort(__float2half_rn(v[k].y * inv)) << 16);
      const uint32_t hi = (uint32_t)__half_as_ushort(__float2half_rn(v[k].z * inv)) |
                          ((uint32_t)__half_as_ushort(__float2half_rn(v[k].w * inv)) << 16);
      *reinterpret_cast<uint2*>(x + row * n + 4 * i) = make_uint2(lo, hi);
    }
  }
}

// qkv[b] = [q (h_q*d) | k (h_kv*d) | v (h_kv*d)] fp32 -> rotated q, k and v in
// fp16 (rope_cos_sin / rope_first / rope_second).
__global__ void rope_split_kernel(const float* __restrict__ qkv, int h_q, int h_kv, int d, int pos,
                                  double theta, uint16_t* __restrict__ q, uint16_t* __restrict__ k,
                                  uint16_t* __restrict__ v) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.y;
  const int head = blockIdx.x;  // 0..h_q+2*h_kv-1
  const int half = d / 2;
  const float* src = qkv + ((long)b * (h_q + 2 * h_kv) + head) * d;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    float x0 = src[i], x1 = src[i + half];
    if (head < h_q + h_kv) {
      float c, s;
      rope_cos_sin(pos, theta, i, d, c, s);
      const float y0 = rope_first(x0, x1, c, s), y1 = rope_second(x0, x1, c, s);
      x0 = y0, x1 = y1;
    }
    uint16_t* dst;
    if (head < h_q)
      dst = q + ((long)b * h_q + head) * d;
    else if (head < h_q + h_kv)
      dst = k + ((long)b * h_kv + head - h_q) * d;
    else
      dst = v + ((long)b * h_kv + head - h_q - h_kv) * d;
    dst[i] = __half_as_ushort(__float2half_rn(x0));
    dst[i + half] = __half_as_ushort(__float2half_rn(x1));
  }
}

// out[b][i] = fp16(silu(gu[b][i]) * gu[b][inter + i])
__global__ void silu_mul_kernel(const float* __restrict__ gu, int inter, uint16_t* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const long b = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < inter; i += gridDim.x * blockDim.x) {
    float g = gu[b * 2 * inter + i], u = gu[b * 2 * inter + inter + i];
    float s = g / (1.0f + expf(-g));
    out[b * inter + i] = __half_as_ushort(__float2half_rn(s * u));
  }
}

__global__ void widen_f16_kernel(const uint16_t* __restrict__ x, long n, float* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    y[i] = h2f(x[i]);
}

__global__ void cast_f16_kernel(const float* __restrict__ x, long n, uint16_t* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    y[i] = __half_as_ushort(__float2half_rn(x[i]));
}

// y[b][i] = sum_c w[i][c] x[b][c], fp16 weights and activations, fp32
// accumulation.  One warp per output row, 16-byte loads, rows strided over
// the grid; x in shared memory as fp32.
template <int BATCH>
__global__ void __launch_bounds__(256) gemv_f16_kernel(const uint16_t* __restrict__ w,
                                                       const uint16_t* __restrict__ x, int n,
                                                       int k, float* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float xs[];  // BATCH * k
  for (int i = threadIdx.x; i < BATCH * k; i += blockDim.x) xs[i] = h2f(x[i]);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < n; row += warps) {
    const uint4* wr = reinterpret_cast<const uint4*>(w + (long)row * k);
    float acc[BATCH];
#pragma unroll
    for (int b = 0; b < BATCH; b++) acc[b] = 0.f;
    for (int c = lane; c < k / 8; c += 32) {
      uint4 v = __ldg(wr + c);
      const __half2* hv = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int e = 0; e < 4; e++) {
        float2 f = __half22float2(hv[e]);
#pragma unroll
        for (int b = 0; b < BATCH; b++) {
          acc[b] = fmaf(f.x, xs[b * k + 8 * c + 2 * e], acc[b]);
          acc[b] = fmaf(f.y, xs[b * k + 8 * c + 2 * e + 1], acc[b]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < BATCH; b++) {
      float v = acc[b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) y[(long)b * n + row] = v;
    }
  }
}

template <int BATCH>
sf_status launch_gemv_f16(const uint16_t* w, const uint16_t* x, int n, int k, float* y, cudaStream_t s) {
  size_t smem = (size_t)BATCH * k * 4;
  SF_CUDA(cudaFuncSetAttribute(gemv_f16_kernel<BATCH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int blocks = 4 * num_sms();
  SF_CUDA(launch_pdl(gemv_f16_kernel<BATCH>, dim3(blocks), dim3(256), smem, s, w, x, n, k, y));
  return SF_OK;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" sf_status sf_rmsnorm_residual(float* h, const float* add0, const float* add1, int batch,
                                         int n, float eps, uint16_t* x, sf_stream_t stream) {
  SF_REQUIRE(h && x && batch > 0 && n > 0, "bad rmsnorm arguments");
  SF_REQUIRE(aligned16(h) && aligned16(x) && (!add0 || aligned16(add0)) && (!add1 || aligned16(add1)),
             "rmsnorm pointers must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  // rows of up to 16,384 elements, a multiple of 4: held in registers
  const int vpt = n % 4 == 0 ? (n / 4 + 1023) / 1024 : 0;
  if (vpt == 1)
    SF_CUDA(launch_pdl(rmsnorm_residual_vec_kernel<1>, dim3(batch), dim3(1024), 0, s, h, add0, add1, n, eps, x));
  else if (vpt == 2)
    SF_CUDA(launch_pdl(rmsnorm_residual_vec_kernel<2>, dim3(batch), dim3(1024), 0, s, h, add0, add1, n, eps, x));
  else if (vpt >= 3 && vpt <= 4)
    SF_CUDA(launch_pdl(rmsnorm_residual_vec_kernel<4>, dim3(batch), dim3(1024), 0, s, h, add0, add1, n, eps, x));
  else
    SF_CUDA(launch_pdl(rmsnorm_residual_kernel, dim3(batch), dim3(1024), 0, s, h, add0, add1, n, eps, x));
  return SF_OK;
}

extern "C" sf_status sf_rope_split(const float* qkv, int batch, int h_q, int h_kv, int d, int pos,
                                   float theta, uint16_t* q, uint16_t* k, uint16_t* v,
                                   sf_stream_t stream) {
  SF_REQUIRE(qkv && q && k && v && batch > 0 && h_q > 0 && h_kv > 0 && d > 0 && d % 2 == 0 && pos >= 0,
             "bad rope arguments");
  SF_CUDA(launch_pdl(rope_split_kernel, dim3(h_q + 2 * h_kv, batch), dim3(64), 0, as_stream(stream), qkv, h_q,
                     h_kv, d, pos, (double)theta, q, k, v));
  return SF_OK;
}

extern "C" sf_status sf_silu_mul(const float* gu, int batch, int inter, uint16_t* out,
                                 sf_stream_t stream) {
  SF_REQUIRE(gu && out && batch > 0 && inter > 0, "bad silu_mul arguments");
  SF_CUDA(launch_pdl(silu_mul_kernel, dim3((inter + 255) / 256, batch), dim3(256), 0, as_stream(stream), gu, inter,
                     out));
  return SF_OK;
}

extern "C" sf_status sf_cast_f16(const float* x, size_t n, uint16_t* y, sf_stream_t stream) {
  SF_REQUIRE(x && y, "bad cast arguments");
  if (n == 0) return SF_OK;
  long blocks = (long)((n + 255) / 256);
  if (blocks > 8 * num_sms()) blocks = 8 * num_sms();
  SF_CUDA(launch_pdl(cast_f16_kernel, dim3((unsigned)blocks), dim3(256), 0, as_stream(stream), x, (long)n, y));
  return SF_OK;
}

extern "C" sf_status sf_widen_f16(const uint16_t* x, size_t n, float* y, sf_stream_t stream) {
  SF_REQUIRE(x && y, "bad widen arguments");
  if (n == 0) return SF_OK;
  long blocks = (long)((n + 255) / 256);
  if (blocks > 8 * num_sms()) blocks = 8 * num_sms();
  SF_CUDA(launch_pdl(widen_f16_kernel, dim3((unsigned)blocks), dim3(256), 0, as_stream(stream), x, (long)n, y));
  return SF_OK;
}

extern "C" sf_status sf_gemv_f16(const uint16_t* w, const uint16_t* x, int batch, int n, int k,
                                 float* y, sf_stream_t stream) {
  SF_REQUIRE(w && x && y && aligned16(w) && aligned16(x) && aligned16(y), "bad gemv_f16 pointers");
  SF_REQUIRE(n > 0 && k > 0 && k % 8 == 0, "k must be a positive multiple of 8");
  SF_UNSUPPORTED(batch >= 1 && batch <= 8 && (size_t)batch * k * 4 <= 200 * 1024,
                 "batch=%d, k=%d too large", batch, k);
  cudaStream_t s = as_stream(stream);
  switch (batch) {
    case 1: return launch_gemv_f16<1>(w, x, n, k, y, s);
    case 2: return launch_gemv_f16<2>(w, x, n, k, y, s);
    case 3: return launch_gemv_f16<3>(w, x, n, k, y, s);
    case 4: return launch_gemv_f16<4>(w, x, n, k, y, s);
    case 5: return launch_gemv_f16<5>(w, x, n, k, y, s);
    case 6: return launch_gemv_f16<6>(w, x, n, k, y, s);
    case 7: return launch_gemv_f16<7>(w, x, n, k, y, s);
    default: return launch_gemv_f16<8>(w, x, n, k, y, s);
  }
}
