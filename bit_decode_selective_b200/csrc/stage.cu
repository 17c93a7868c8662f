// stage.cu -- staging of selected refinement rows from pinned host memory.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?": on a
// machine with a dedicated GPU the refinement bits live in host RAM; only the
// rows of the selected channels cross the link, and fetch lead starts that
// transfer one or more layers early, from an earlier activation, so it
// overlaps the projections in between.
//
// sf_stage_refinements gathers the rows named by a DEVICE index array straight
// from mapped pinned host memory (the GPU issues the PCIe reads itself), so a
// selection made on the GPU needs no round trip through the host and the copy
// can be captured in a CUDA graph.  sf_stage_refinements_host is the plain
// variant for indices known on the host: one cudaMemcpyAsync per run of
// consecutive rows.
#include "common.cuh"

namespace sf {
namespace {

constexpr int kVec = 4;                // 16-byte words in flight per thread
constexpr int kGatherThreads = 128;     // small CTAs: each fits in the room whole-SM kernels leave
constexpr int kGatherBlocksMax = 64;    // 64 x 8 KB in flight keeps the host link busy

// CTAs walk the n_sel x row_vecs 16-byte words of the selected rows, kVec loads
// in flight per thread.  The reads cross the host link, so the CTAs live about
// as long as the transfer; each fits beside a whole-SM kernel's CTA (at most
// kSideRegs registers, no shared memory), so the transfer never delays one.
static_assert(kGatherThreads * 32 <= kSideRegs, "a gather CTA must fit in the room left for staging");
// An index outside [0, n_rows) is never dereferenced: its row is filled with
// zeros and counted in *bad (when given), which the host can read back.
__global__ void __maxnreg__(32) gather_rows_kernel(const uint4* __restrict__ src, size_t row_vecs,
                                                   const int32_t* __restrict__ sel, int n_sel, int n_rows,
                                                   uint4* __restrict__ dst, int32_t* __restrict__ bad) {
  const size_t total = (size_t)n_sel * row_vecs;
  const size_t step = (size_t)gridDim.x * kGatherThreads * kVec;
  for (size_t base = (size_t)blockIdx.x * kGatherThreads * kVec + threadIdx.x; base < total; base += step) {
    uint4 v[kVec];
#pragma unroll
    for (int u = 0; u < kVec; u++) {
      const size_t i = base + (size_t)u * kGatherThreads;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i < total) {
        const size_t j = i / row_vecs, c = i - j * row_vecs;
        const int32_t row = sel[j];
        if (row >= 0 && row < n_rows) {
          v[u] = src[(size_t)row * row_vecs + c];
        } else if (bad && c == 0) {
          atomicAdd(bad, 1);  // once per bad index
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kVec; u++) {
      const size_t i = base + (size_t)u * kGatherThreads;
      if (i < total) dst[i] = v[u];
    }
  }
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" sf_status sf_stage_refinements(const void* host_rows, size_t row_bytes, int n_rows,
                                          const int32_t* sel, int n_sel, void* dst, int32_t* bad,
                                          sf_stream_t stream, sf_event_t done) {
  SF_REQUIRE(host_rows && dst && sel, "host_rows, sel and dst must be non-null");
  SF_REQUIRE(n_rows >= 1, "n_rows=%d < 1", n_rows);
  SF_REQUIRE(!bad || (reinterpret_cast<uintptr_t>(bad) & 3u) == 0, "bad must be 4-byte aligned");
  SF_REQUIRE(row_bytes > 0 && row_bytes % 16 == 0, "row_bytes=%zu must be a multiple of 16",
             row_bytes);
  SF_REQUIRE(aligned16(host_rows) && aligned16(dst) && aligned16(sel),
             "host_rows, sel and dst must be 16-byte aligned");
  SF_REQUIRE(n_sel >= 0, "n_sel=%d < 0", n_sel);
  cudaPointerAttributes attr;
  SF_CUDA(cudaPointerGetAttributes(&attr, host_rows));
  SF_REQUIRE(attr.type == cudaMemoryTypeHost && attr.devicePointer != nullptr,
             "host_rows must be page-locked host memory mapped into the device address space");
  cudaStream_t s = as_stream(stream);
  if (n_sel > 0) {
    const size_t vecs = (size_t)n_sel * (row_bytes / 16);
    size_t blocks = (vecs + kGatherThreads * kVec - 1) / (kGatherThreads * kVec);
    if (blocks > (size_t)kGatherBlocksMax) blocks = kGatherBlocksMax;
    gather_rows_kernel<<<(unsigned)blocks, kGatherThreads, 0, s>>>((const uint4*)attr.devicePointer,
                                                                   (size_t)(row_bytes / 16), sel, n_sel, n_rows,
                                                                   (uint4*)dst, bad);
    SF_LAUNCHED();
  }
  if (done) SF_CUDA(cudaEventRecord((cudaEvent_t)done, s));
  return SF_OK;
}

extern "C" sf_status sf_stage_refinements_host(const void* host_rows, size_t row_bytes, int n_rows,
                                               const int32_t* sel_host, int n_sel, void* dst,
                                               sf_stream_t stream, sf_event_t done) {
  SF_REQUIRE(host_rows && dst && (sel_host || n_sel == 0), "null argument");
  SF_REQUIRE(row_bytes > 0, "row_bytes must be positive");
  SF_REQUIRE(n_sel >= 0, "n_sel=%d < 0", n_sel);
  SF_REQUIRE(n_rows >= 1, "n_rows=%d < 1", n_rows);
  for (int j = 0; j < n_sel; j++)  // every index is checked before anything is enqueued
    SF_REQUIRE(sel_host[j] >= 0 && sel_host[j] < n_rows, "row index %d (entry %d) outside [0, %d)",
               sel_host[j], j, n_rows);
  cudaStream_t s = as_stream(stream);
  const char* src = (const char*)host_rows;
  char* out = (char*)dst;
  int j = 0;
  while (j < n_sel) {
    int run = 1;
    while (j + run < n_sel && sel_host[j + run] == sel_host[j] + run) run++;
    SF_CUDA(cudaMemcpyAsync(out + (size_t)j * row_bytes, src + (size_t)sel_host[j] * row_bytes,
                            (size_t)run * row_bytes, cudaMemcpyHostToDevice, s));
    j += run;
  }
  if (done) SF_CUDA(cudaEventRecord((cudaEvent_t)done, s));
  return SF_OK;
}
