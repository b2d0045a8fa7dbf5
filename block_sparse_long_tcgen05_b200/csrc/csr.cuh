// Block -> query inverted index (CSR), built by a stable counting sort.
//
// KV-outer execution (hyper.ai "MiniMax Sparse Attention", Key Contributions; zhichai.net
// section 4.2 "KV-outer") keeps one K/V block on chip and streams the queries that chose
// it, so each (group g, block b) needs the list of (query i, slot s) pairs whose
// block_ids[i, g, s] == b. This file builds that list for the queries of one chunk:
//
//   1. csr_count:   per (query block qt, group): a 128-bit membership mask per block b
//                   (which of the tile's 128 queries chose b); its popcount goes to
//                   hist[g, b, qt];
//   2. csr_scan:    exclusive scan of hist[g, b, :] over the tiles -> in place, and the
//                   bucket totals;
//   3. csr_offsets: exclusive scan of the totals over all (g, b) -> bucket starts, and
//                   of the KV-outer work items per bucket -> item starts;
//   4. csr_scatter: each query writes (i << 5 | s) at bucket start + tile offset + its
//                   rank among the tile's queries in that bucket (popcount of the mask
//                   below it), so every bucket lists its queries in ascending order
//                   (deterministic, no atomics on the output);
//   5. csr_items:   cut every bucket into work items of at most kItemTiles tiles.
#pragma once
#include "ptx.cuh"

namespace msa {

struct CsrParams {
  const int32_t* block_ids;  // [N, G, k]
  int64_t N;
  int G, k;
  int qa0, qa1;              // query blocks of this chunk; buckets cover blocks [0, qa1)
  int nt;                    // qa1 - qa0
  int tq;                    // queries per KV-outer tile
  int item_tiles;            // tiles per work item
  uint32_t* hist;            // [G, qa1, nt]
  uint32_t* totals;          // [G * qa1]
  uint32_t* bucket_start;    // [G * qa1 + 1]
  uint32_t* item_start;      // [G * qa1 + 1]
  int32_t* entries;          // [sum of totals]
  int4* items;               // [n_items]
};

// The ids of a row are accepted when they are -1 padded at the end, strictly
// ascending, and each lies in [0, bl]. Otherwise the row is dropped (no output) and
// MSA_ERR_DEVICE_BOUNDS is recorded.
__device__ __forceinline__ bool csr_row_valid(const int32_t* ids, int k, int bl) {
  int prev = -1;
  bool ended = false;
  for (int s = 0; s < k; ++s) {
    const int b = ids[s];
    if (b < 0) {
      if (b != -1) return false;
      ended = true;
      continue;
    }
    if (ended || b <= prev || b > bl) return false;
    prev = b;
  }
  return true;
}

// builds the membership masks of query block qb for group g into smem bm[(qb+1)*4]
__device__ __forceinline__ void csr_build_masks(const CsrParams& P, int qb, int g, uint32_t* bm, int32_t* my_ids,
                                                bool& row_ok) {
  const int r = threadIdx.x;
  for (int w = r; w < (qb + 1) * 4; w += blockDim.x) bm[w] = 0u;
  __syncthreads();
  const int64_t i = static_cast<int64_t>(qb) * 128 + r;
  row_ok = false;
  if (i < P.N) {
    const int32_t* src = P.block_ids + (i * P.G + g) * P.k;
    for (int s = 0; s < P.k; ++s) my_ids[s] = src[s];
    row_ok = csr_row_valid(my_ids, P.k, qb);
    if (!row_ok) record_error(MSA_ERR_DEVICE_BOUNDS, kKidCsr);
    if (row_ok)
      for (int s = 0; s < P.k; ++s)
        if (my_ids[s] >= 0) atomicOr(&bm[my_ids[s] * 4 + (r >> 5)], 1u << (r & 31));
  }
  __syncthreads();
}

__global__ void __launch_bounds__(128) csr_count_kernel(const __grid_constant__ CsrParams P) {
  extern __shared__ uint32_t bm[];
  const int qt = blockIdx.x, g = blockIdx.y;
  const int qb = P.qa0 + qt;
  int32_t ids[32];
  bool ok;
  csr_build_masks(P, qb, g, bm, ids, ok);
  for (int b = threadIdx.x; b <= qb; b += blockDim.x) {
    const uint32_t c = __popc(bm[b * 4 + 0]) + __popc(bm[b * 4 + 1]) + __popc(bm[b * 4 + 2]) + __popc(bm[b * 4 + 3]);
    P.hist[(static_cast<int64_t>(g) * P.qa1 + b) * P.nt + qt] = c;
  }
}

// one warp per bucket (g, b); tiles before b's own query block cannot choose b
__global__ void __launch_bounds__(256) csr_scan_kernel(const __grid_constant__ CsrParams P) {
  const int64_t bucket = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bucket >= static_cast<int64_t>(P.G) * P.qa1) return;
  const int b = static_cast<int>(bucket % P.qa1);
  const int t0 = max(0, b - P.qa0);
  uint32_t* h = P.hist + bucket * P.nt;
  uint32_t run = 0;
  for (int base = t0; base < P.nt; base += 32) {
    const int t = base + lane;
    const uint32_t v = (t < P.nt) ? h[t] : 0u;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (t < P.nt) h[t] = run + x - v;
    run += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) P.totals[bucket] = run;
}

// single CTA of 1024 threads: exclusive scans over all buckets
__global__ void __launch_bounds__(1024) csr_offsets_kernel(const __grid_constant__ CsrParams P) {
  __shared__ uint32_t s_e[32], s_i[32];
  const int nbuck = P.G * P.qa1;
  const int per = (nbuck + 1023) / 1024;
  const int lo = min(nbuck, threadIdx.x * per), hi = min(nbuck, lo + per);
  const uint32_t tile_q = static_cast<uint32_t>(P.tq) * static_cast<uint32_t>(P.item_tiles);
  uint32_t se = 0, si = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t t = P.totals[j];
    se += t;
    si += (t + tile_q - 1) / tile_q;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t xe = se, xi = si;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t ye = __shfl_up_sync(0xffffffffu, xe, o), yi = __shfl_up_sync(0xffffffffu, xi, o);
    if (lane >= o) { xe += ye; xi += yi; }
  }
  if (lane == 31) { s_e[warp] = xe; s_i[warp] = xi; }
  __syncthreads();
  if (warp == 0) {
    uint32_t ve = s_e[lane], vi = s_i[lane];
    uint32_t ae = ve, ai = vi;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t ye = __shfl_up_sync(0xffffffffu, ae, o), yi = __shfl_up_sync(0xffffffffu, ai, o);
      if (lane >= o) { ae += ye; ai += yi; }
    }
    s_e[lane] = ae - ve;
    s_i[lane] = ai - vi;
  }
  __syncthreads();
  uint32_t oe = s_e[warp] + xe - se, oi = s_i[warp] + xi - si;
  for (int j = lo; j < hi; ++j) {
    const uint32_t t = P.totals[j];
    P.bucket_start[j] = oe;
    P.item_start[j] = oi;
    oe += t;
    oi += (t + tile_q - 1) / tile_q;
  }
  if (threadIdx.x == 1023) {
    P.bucket_start[nbuck] = oe;
    P.item_start[nbuck] = oi;
  }
}

__global__ void __launch_bounds__(128) csr_scatter_kernel(const __grid_constant__ CsrParams P) {
  extern __shared__ uint32_t bm[];
  const int qt = blockIdx.x, g = blockIdx.y;
  const int qb = P.qa0 + qt;
  int32_t ids[32];
  bool ok;
  csr_build_masks(P, qb, g, bm, ids, ok);
  if (!ok) return;
  const int r = threadIdx.x;
  const int64_t i = static_cast<int64_t>(qb) * 128 + r;
  const uint32_t below = (1u << (r & 31)) - 1u;
  for (int s = 0; s < P.k; ++s) {
    const int b = ids[s];
    if (b < 0) break;
    const uint32_t* m = bm + b * 4;
    uint32_t rank = __popc(m[r >> 5] & below);
    for (int w = 0; w < (r >> 5); ++w) rank += __popc(m[w]);
    const int64_t bucket = static_cast<int64_t>(g) * P.qa1 + b;
    const uint32_t pos = P.bucket_start[bucket] + P.hist[bucket * P.nt + qt] + rank;
    P.entries[pos] = static_cast<int32_t>((i << 5) | s);
  }
}

__global__ void __launch_bounds__(256) csr_items_kernel(const __grid_constant__ CsrParams P) {
  const int64_t bucket = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (bucket >= static_cast<int64_t>(P.G) * P.qa1) return;
  const uint32_t tot = P.totals[bucket];
  const uint32_t e0 = P.bucket_start[bucket];
  uint32_t it = P.item_start[bucket];
  const uint32_t per = static_cast<uint32_t>(P.tq) * static_cast<uint32_t>(P.item_tiles);
  for (uint32_t off = 0; off < tot; off += per, ++it)
    P.items[it] = make_int4(static_cast<int>(bucket), static_cast<int>(e0 + off), static_cast<int>(min(per, tot - off)), 0);
}

}  // namespace msa
