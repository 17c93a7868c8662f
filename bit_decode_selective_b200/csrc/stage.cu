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


// ---- a device-resident cache of refinement rows, reused across steps
//
// [EXPL] "the map app also loads tiles": bits fetched for one step are kept
// and reused while the selection repeats; on a miss the runtime either waits
// for the transfer or runs the channel at its resident precision for now.
//
// cache_book_kernel (one CTA): marks the selected channels the cache holds as
// used in this step, gives every missing channel a slot (the slots not used in
// this step, in clock order from the hand: least recently reused first) and
// writes, per entry, the source (a slot of the cache, or -1 - the slot a
// missing row goes to) and the effective selection.  Rows then move with
// cache_gather_kernel: hits from the cache, misses from host memory into their
// slot (and into the staging slot when the caller waits for them).

constexpr int kBookThreads = 1024;
constexpr int kCacheCapMax = 8192;
constexpr int kCacheSelMax = 4096;
constexpr int kCacheBatchMax = 8;

struct CacheSet {
  sf_row_cache c[kCacheBatchMax];  // one cache per batch row
};

// One CTA per batch row.
__global__ void __launch_bounds__(kBookThreads) cache_book_kernel(CacheSet cs, const int32_t* __restrict__ sel_all,
                                                                  int n_sel, int skip, int32_t* __restrict__ eff_all) {
  __shared__ int ws[40];
  __shared__ int vict[kCacheSelMax];
  __shared__ uint32_t now_s, hand_s;
  __shared__ int hits_s;
  const sf_row_cache& c = cs.c[blockIdx.x];
  const int32_t* sel = sel_all + (size_t)blockIdx.x * n_sel;
  int32_t* sel_eff = eff_all + (size_t)blockIdx.x * n_sel;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    now_s = c.state[0] + 1u;
    hand_s = c.state[1];
    hits_s = 0;
  }
  __syncthreads();
  const uint32_t now = now_s;
  constexpr int PER = kCacheSelMax / kBookThreads;
  int ch[PER], slot[PER];
  bool miss[PER];
  int nmiss = 0, nhit = 0;
#pragma unroll
  for (int u = 0; u < PER; u++) {
    const int j = tid * PER + u;
    ch[u] = -1, slot[u] = -1, miss[u] = false;
    if (j < n_sel) {
      const int cc = sel[j];
      if (cc >= 0 && cc < c.n_channels) {  // an index outside the cache's channels is never staged
        ch[u] = cc;
        slot[u] = c.slot_of[cc];
        miss[u] = slot[u] < 0;
        if (!miss[u]) c.stamp[slot[u]] = now, nhit++;
        else nmiss++;
      }
    }
  }
  auto excl = [&](int v, int& total) {  // exclusive prefix over the threads, in thread order
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    __syncthreads();
    if (lane == 31) ws[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wv = ws[lane];
      int x = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
      }
      ws[lane] = x - wv;
      if (lane == 31) ws[32] = x;
    }
    __syncthreads();
    total = ws[32];
    return ws[warp] + incl - v;
  };
  int misses;
  const int rank0 = excl(nmiss, misses);  // (its barriers also order the stamps of the hits)
  // the slots not used in this step, in clock order from the hand
  const int cap = c.capacity;
  const int sper = (cap + kBookThreads - 1) / kBookThreads;
  int nfree = 0;
  for (int i = tid * sper; i < min(cap, (tid + 1) * sper); i++)
    nfree += c.stamp[(int)((hand_s + (uint32_t)i) % (uint32_t)cap)] != now;
  int frees;
  int r = excl(nfree, frees);
  for (int i = tid * sper; i < min(cap, (tid + 1) * sper); i++) {
    const int s = (int)((hand_s + (uint32_t)i) % (uint32_t)cap);
    if (c.stamp[s] != now) {
      if (r < misses) vict[r] = s;
      r++;
    }
  }
  __syncthreads();
  // the missing channels take their slots
  int k = rank0;
#pragma unroll
  for (int u = 0; u < PER; u++) {
    const int j = tid * PER + u;
    if (j >= n_sel) continue;
    if (ch[u] < 0) {
      c.work[j] = 0x7fffffff;  // nothing to move
      sel_eff[j] = -1 - max(0, min(sel[j], c.n_channels - 1));
    } else if (miss[u]) {
      const int v = vict[k++];
      const int old = c.channel_of[v];
      if (old >= 0) c.slot_of[old] = -1;
      c.channel_of[v] = ch[u];
      c.slot_of[ch[u]] = v;
      c.stamp[v] = now;
      c.work[j] = -1 - v;
      sel_eff[j] = skip ? -1 - ch[u] : ch[u];
    } else {
      c.work[j] = slot[u];
      sel_eff[j] = ch[u];
    }
  }
  if (nhit) atomicAdd(&hits_s, nhit);
  __syncthreads();
  if (tid == 0) {
    c.state[0] = now;
    if (misses > 0) c.state[1] = (uint32_t)((vict[misses - 1] + 1) % cap);
    c.state[2] += (uint32_t)hits_s;
    c.state[3] += (uint32_t)misses;
  }
}

// Rows of every batch row's entries: mode 0 all of them into dst (hits from
// the cache, misses from host memory, also written into their slot); mode 1
// hits only; mode 2 misses into their slots only.
__global__ void __maxnreg__(32) cache_gather_kernel(CacheSet cs, const uint4* __restrict__ host, size_t row_vecs,
                                                    const int32_t* __restrict__ sel, int n_sel, int batch,
                                                    uint4* __restrict__ dst, int mode) {
  const size_t per_b = (size_t)n_sel * row_vecs;
  const size_t total = per_b * batch;
  const size_t step = (size_t)gridDim.x * kGatherThreads * kVec;
  for (size_t base = (size_t)blockIdx.x * kGatherThreads * kVec + threadIdx.x; base < total; base += step) {
    uint4 v[kVec];
    int w[kVec];
#pragma unroll
    for (int u = 0; u < kVec; u++) {
      const size_t i = base + (size_t)u * kGatherThreads;
      w[u] = 0x7fffffff;  // nothing to move
      if (i < total) {
        const int b = (int)(i / per_b);
        const size_t ib = i - (size_t)b * per_b, j = ib / row_vecs, cv = ib - j * row_vecs;
        const int wj = cs.c[b].work[j];
        if (wj >= 0 && wj != 0x7fffffff && mode != 2) {
          w[u] = wj, v[u] = reinterpret_cast<const uint4*>(cs.c[b].rows)[(size_t)wj * row_vecs + cv];
        } else if (wj < 0 && mode != 1) {
          w[u] = wj, v[u] = host[(size_t)sel[(size_t)b * n_sel + j] * row_vecs + cv];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kVec; u++) {
      if (w[u] == 0x7fffffff) continue;
      const size_t i = base + (size_t)u * kGatherThreads;
      if (w[u] >= 0) {
        dst[i] = v[u];
      } else {
        const int b = (int)(i / per_b);
        const size_t ib = i - (size_t)b * per_b, j = ib / row_vecs;
        reinterpret_cast<uint4*>(cs.c[b].rows)[(size_t)(-1 - w[u]) * row_vecs + (ib - j * row_vecs)] = v[u];
        if (mode == 0) dst[i] = v[u];
      }
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

extern "C" sf_status sf_row_cache_reset(const sf_row_cache* c, sf_stream_t stream) {
  SF_REQUIRE(c && c->slot_of && c->channel_of && c->stamp && c->state, "null cache arrays");
  cudaStream_t s = as_stream(stream);
  SF_CUDA(cudaMemsetAsync(c->slot_of, 0xff, (size_t)c->n_channels * 4, s));
  SF_CUDA(cudaMemsetAsync(c->channel_of, 0xff, (size_t)c->capacity * 4, s));
  SF_CUDA(cudaMemsetAsync(c->stamp, 0, (size_t)c->capacity * 4, s));
  SF_CUDA(cudaMemsetAsync(c->state, 0, 4 * 4, s));
  return SF_OK;
}

extern "C" sf_status sf_stage_refinements_cached(const void* host_rows, size_t row_bytes, int n_rows,
                                                 const int32_t* sel, int n_sel, int batch,
                                                 const sf_row_cache* caches, int skip_missing, void* dst,
                                                 int32_t* sel_eff, sf_stream_t stream, sf_event_t done) {
  SF_REQUIRE(host_rows && dst && sel && sel_eff && caches, "host_rows, sel, caches, dst and sel_eff must be non-null");
  SF_REQUIRE(row_bytes > 0 && row_bytes % 16 == 0, "row_bytes=%zu must be a multiple of 16", row_bytes);
  SF_REQUIRE(aligned16(host_rows) && aligned16(dst) && aligned16(sel) && aligned16(sel_eff),
             "host_rows, sel, sel_eff and dst must be 16-byte aligned");
  SF_REQUIRE(n_sel >= 0, "n_sel=%d < 0", n_sel);
  SF_UNSUPPORTED(batch >= 1 && batch <= kCacheBatchMax, "batch=%d outside [1, %d]", batch, kCacheBatchMax);
  SF_UNSUPPORTED(n_sel <= kCacheSelMax, "n_sel=%d above %d", n_sel, kCacheSelMax);
  CacheSet cs = {};
  for (int b = 0; b < batch; b++) {
    const sf_row_cache& c = caches[b];
    SF_REQUIRE(c.slot_of && c.channel_of && c.stamp && c.state && c.work && c.rows && aligned16(c.rows),
               "null or misaligned arrays in cache %d", b);
    SF_REQUIRE(c.row_bytes == (int)row_bytes, "cache %d holds rows of %d bytes, staging rows of %zu", b,
               c.row_bytes, row_bytes);
    SF_REQUIRE(c.n_channels == n_rows, "cache %d indexes %d channels, host_rows holds %d rows", b, c.n_channels,
               n_rows);
    SF_UNSUPPORTED(c.capacity >= 1 && c.capacity <= kCacheCapMax, "capacity %d outside [1, %d]", c.capacity,
                   kCacheCapMax);
    SF_REQUIRE(n_sel <= c.capacity && n_sel <= c.max_sel, "n_sel=%d above cache %d's capacity %d or max_sel %d",
               n_sel, b, c.capacity, c.max_sel);
    cs.c[b] = c;
  }
  cudaPointerAttributes attr;
  SF_CUDA(cudaPointerGetAttributes(&attr, host_rows));
  SF_REQUIRE(attr.type == cudaMemoryTypeHost && attr.devicePointer != nullptr,
             "host_rows must be page-locked host memory mapped into the device address space");
  cudaStream_t s = as_stream(stream);
  const size_t vecs = (size_t)batch * n_sel * (row_bytes / 16);
  size_t blocks = (vecs + kGatherThreads * kVec - 1) / (kGatherThreads * kVec);
  if (blocks > (size_t)kGatherBlocksMax) blocks = kGatherBlocksMax;
  if (n_sel > 0) {
    cache_book_kernel<<<batch, kBookThreads, 0, s>>>(cs, sel, n_sel, skip_missing ? 1 : 0, sel_eff);
    SF_LAUNCHED();
    cache_gather_kernel<<<(unsigned)blocks, kGatherThreads, 0, s>>>(cs, (const uint4*)attr.devicePointer,
                                                                    row_bytes / 16, sel, n_sel, batch, (uint4*)dst,
                                                                    skip_missing ? 1 : 0);
    SF_LAUNCHED();
  }
  if (done) SF_CUDA(cudaEventRecord((cudaEvent_t)done, s));
  if (n_sel > 0 && skip_missing) {  // the missing rows land in the cache after `done`
    cache_gather_kernel<<<(unsigned)blocks, kGatherThreads, 0, s>>>(cs, (const uint4*)attr.devicePointer,
                                                                    row_bytes / 16, sel, n_sel, batch, (uint4*)dst, 2);
    SF_LAUNCHED();
  }
  return SF_OK;
}
