// Block -> query inverted index (CSR), built by a stable counting sort.
//
// KV-outer execution (hyper.ai "MiniMax Sparse Attention", Key Contributions; zhichai.net
// section 4.2 "KV-outer") keeps one K/V block on chip and streams the queries that chose
// it, so each (group g, block b) needs the list of (query i, slot s) pairs whose
// block_ids[i, g, s] == b. The Main Branch runs in query chunks of CT tiles of 128 queries;
// this file builds the lists of every chunk at once, each chunk in its own region, in five
// launches per forward:
//
//   1. csr_count:   per (query tile t, group): a 128-bit membership mask per block b that
//                   the tile can see (which of its 128 queries chose b); its popcount goes
//                   to hist[g, b, t] of the tile's chunk;
//   2. csr_scan:    per bucket (chunk, g, b): exclusive scan of hist[g, b, :] over the
//                   chunk's tiles -> in place, and the bucket totals;
//   3. csr_offsets: per chunk, exclusive scans of the totals over all its (g, b) -> bucket
//                   starts, and of the KV-outer work items per bucket -> item starts;
//   4. csr_scatter: each query writes (i << 5 | s) at bucket start + tile offset + its
//                   rank among the tile's queries in that bucket (popcount of the mask
//                   below it), so every bucket lists its queries in ascending order
//                   (deterministic, no atomics on the output);
//   5. csr_items:   cut every bucket into work items of at most item_tiles tiles.
//
// Blocks hold bk tokens, bk in {32, 64, 128}; a 128-query tile sees bpt = 128 / bk blocks of
// its own span, so tile t sees blocks [0, (t + 1) * bpt).
#pragma once
#include "ptx.cuh"

namespace msa {

constexpr int kCsrMaxChunks = 128;

// Per-chunk offsets of the chunk's regions in the shared arrays (computed on the host).
struct CsrChunkTable {
  int64_t hist[kCsrMaxChunks];          // uint32 entries of hist before the chunk
  int64_t bucket[kCsrMaxChunks + 1];    // buckets before the chunk (totals, and G*nbk + 1 slots of bstart/istart)
  int64_t entry[kCsrMaxChunks];         // entries before the chunk
  int64_t item[kCsrMaxChunks];          // work items before the chunk
};

struct CsrParams {
  const int32_t* block_ids;  // [N, G, k]
  int64_t N;
  int G, k;
  int bk, bpt;               // tokens per block, blocks per 128-query tile
  int ntiles;                // 128-query tiles of the sequence
  int nblocks;               // blocks of the sequence, ceil(N / bk)
  int ct;                    // tiles per chunk
  int nchunks;
  int tq;                    // queries per KV-outer tile
  int item_tiles;            // KV-outer tiles per work item
  uint32_t* hist;            // per chunk [G, nbk_c, nt_c]
  uint32_t* totals;          // per chunk [G * nbk_c]
  uint32_t* bucket_start;    // per chunk [G * nbk_c + 1] (at bucket offset + chunk index)
  uint32_t* item_start;      // per chunk [G * nbk_c + 1]
  int32_t* entries;          // per chunk [sum of its totals]
  int4* items;               // per chunk [its items]
};

// Shape of chunk c: first tile, tiles, blocks visible to its last tile.
struct CsrChunk {
  int t0, nt, nbk;
};
__device__ __forceinline__ CsrChunk csr_chunk(const CsrParams& P, int c) {
  CsrChunk ch;
  ch.t0 = c * P.ct;
  ch.nt = min(P.ct, P.ntiles - ch.t0);
  ch.nbk = min(P.nblocks, (ch.t0 + ch.nt) * P.bpt);
  return ch;
}

// The ids of a row are accepted when they are -1 padded at the end, strictly
// ascending, and each lies in [0, bl]. Otherwise the row is dropped (no output) and
// MSA_ERR_DEVICE_BOUNDS is recorded.
// (Loops over the 32 possible slots are unrolled with the row's k as a predicate, so the
// ids stay in registers.)
__device__ __forceinline__ bool csr_row_valid(const int32_t (&ids)[32], int k, int bl) {
  int prev = -1;
  bool ended = false, ok = true;
#pragma unroll
  for (int s = 0; s < 32; ++s) {
    if (s < k) {
      const int b = ids[s];
      if (b < 0) {
        ok = ok && (b == -1);
        ended = true;
      } else {
        ok = ok && !ended && b > prev && b <= bl;
        prev = b;
      }
    }
  }
  return ok;
}

// builds the membership masks of query tile t for group g into smem bm[nbv * 4], nbv the
// blocks tile t can see
__device__ __forceinline__ void csr_build_masks(const CsrParams& P, int t, int nbv, int g, uint32_t* bm,
                                                int32_t (&my_ids)[32], bool& row_ok) {
  const int r = threadIdx.x;
  for (int w = r; w < nbv * 4; w += blockDim.x) bm[w] = 0u;
  __syncthreads();
  const int64_t i = static_cast<int64_t>(t) * 128 + r;
  row_ok = false;
#pragma unroll
  for (int s = 0; s < 32; ++s) my_ids[s] = -1;
  if (i < P.N) {
    const int32_t* src = P.block_ids + (i * P.G + g) * P.k;
#pragma unroll
    for (int s = 0; s < 32; ++s)
      if (s < P.k) my_ids[s] = src[s];
    row_ok = csr_row_valid(my_ids, P.k, static_cast<int>(i / P.bk));
    if (!row_ok) record_error(MSA_ERR_DEVICE_BOUNDS, kKidCsr);
    if (row_ok) {
#pragma unroll
      for (int s = 0; s < 32; ++s)
        if (s < P.k && my_ids[s] >= 0) atomicOr(&bm[my_ids[s] * 4 + (r >> 5)], 1u << (r & 31));
    }
  }
  __syncthreads();
}

// grid (ntiles, G), 128 threads
__global__ void __launch_bounds__(128) csr_count_kernel(const __grid_constant__ CsrParams P,
                                                        const __grid_constant__ CsrChunkTable T) {
  extern __shared__ uint32_t bm[];
  const int t = blockIdx.x, g = blockIdx.y;
  const int c = t / P.ct;
  const CsrChunk ch = csr_chunk(P, c);
  const int qt = t - ch.t0;
  const int nbv = min(P.nblocks, (t + 1) * P.bpt);
  int32_t ids[32];
  bool ok;
  csr_build_masks(P, t, nbv, g, bm, ids, ok);
  uint32_t* hist = P.hist + T.hist[c];
  for (int b = threadIdx.x; b < nbv; b += blockDim.x) {
    const uint32_t n = __popc(bm[b * 4 + 0]) + __popc(bm[b * 4 + 1]) + __popc(bm[b * 4 + 2]) + __popc(bm[b * 4 + 3]);
    hist[(static_cast<int64_t>(g) * ch.nbk + b) * ch.nt + qt] = n;
  }
}

// chunk of flattened bucket u (buckets of all chunks, in chunk order)
__device__ __forceinline__ int csr_bucket_chunk(const CsrParams& P, const CsrChunkTable& T, int64_t u) {
  int lo = 0, hi = P.nchunks - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (T.bucket[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// one warp per bucket (chunk, g, b); tiles before b's own tile cannot choose b
__global__ void __launch_bounds__(256) csr_scan_kernel(const __grid_constant__ CsrParams P,
                                                       const __grid_constant__ CsrChunkTable T) {
  const int64_t u = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (u >= T.bucket[P.nchunks]) return;
  const int c = csr_bucket_chunk(P, T, u);
  const CsrChunk ch = csr_chunk(P, c);
  const int64_t bucket = u - T.bucket[c];                 // g * nbk + b within the chunk
  const int b = static_cast<int>(bucket % ch.nbk);
  const int q0 = max(0, b / P.bpt - ch.t0);
  uint32_t* h = P.hist + T.hist[c] + bucket * ch.nt;
  uint32_t run = 0;
  for (int base = q0; base < ch.nt; base += 32) {
    const int t = base + lane;
    const uint32_t v = (t < ch.nt) ? h[t] : 0u;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (t < ch.nt) h[t] = run + x - v;
    run += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) P.totals[u] = run;
}

// one CTA of 1024 threads per chunk: exclusive scans over the chunk's buckets
__global__ void __launch_bounds__(1024) csr_offsets_kernel(const __grid_constant__ CsrParams P,
                                                           const __grid_constant__ CsrChunkTable T) {
  __shared__ uint32_t s_e[32], s_i[32];
  const int c = blockIdx.x;
  const int nbuck = static_cast<int>(T.bucket[c + 1] - T.bucket[c]);
  const uint32_t* totals = P.totals + T.bucket[c];
  uint32_t* bstart = P.bucket_start + T.bucket[c] + c;
  uint32_t* istart = P.item_start + T.bucket[c] + c;
  const int per = (nbuck + 1023) / 1024;
  const int lo = min(nbuck, static_cast<int>(threadIdx.x) * per), hi = min(nbuck, lo + per);
  const uint32_t tile_q = static_cast<uint32_t>(P.tq) * static_cast<uint32_t>(P.item_tiles);
  uint32_t se = 0, si = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t t = totals[j];
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
    const uint32_t t = totals[j];
    bstart[j] = oe;
    istart[j] = oi;
    oe += t;
    oi += (t + tile_q - 1) / tile_q;
  }
  if (threadIdx.x == 1023) {
    bstart[nbuck] = oe;
    istart[nbuck] = oi;
  }
}

// grid (ntiles, G), 128 threads
__global__ void __launch_bounds__(128) csr_scatter_kernel(const __grid_constant__ CsrParams P,
                                                          const __grid_constant__ CsrChunkTable T) {
  extern __shared__ uint32_t bm[];
  const int t = blockIdx.x, g = blockIdx.y;
  const int c = t / P.ct;
  const CsrChunk ch = csr_chunk(P, c);
  const int qt = t - ch.t0;
  const int nbv = min(P.nblocks, (t + 1) * P.bpt);
  int32_t ids[32];
  bool ok;
  csr_build_masks(P, t, nbv, g, bm, ids, ok);
  if (!ok) return;
  const int r = threadIdx.x;
  const int64_t i = static_cast<int64_t>(t) * 128 + r;
  const uint32_t below = (1u << (r & 31)) - 1u;
  const uint32_t* hist = P.hist + T.hist[c];
  const uint32_t* bstart = P.bucket_start + T.bucket[c] + c;
  int32_t* entries = P.entries + T.entry[c];
  // the bucket starts and tile offsets of all of the row's slots are loaded before any is
  // used (one memory round trip), then each slot's entry goes to its place
  uint32_t base[32];
#pragma unroll
  for (int s = 0; s < 32; ++s) {
    base[s] = 0u;
    if (s < P.k && ids[s] >= 0) {
      const int64_t bucket = static_cast<int64_t>(g) * ch.nbk + ids[s];
      base[s] = __ldg(bstart + bucket) + __ldg(hist + bucket * ch.nt + qt);
    }
  }
#pragma unroll
  for (int s = 0; s < 32; ++s) {
    if (s < P.k && ids[s] >= 0) {
      const uint32_t* m = bm + ids[s] * 4;
      uint32_t rank = __popc(m[r >> 5] & below);
      for (int w = 0; w < (r >> 5); ++w) rank += __popc(m[w]);
      entries[base[s] + rank] = static_cast<int32_t>((i << 5) | s);
    }
  }
}

// one thread per bucket (chunk, g, b)
__global__ void __launch_bounds__(256) csr_items_kernel(const __grid_constant__ CsrParams P,
                                                        const __grid_constant__ CsrChunkTable T) {
  const int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (u >= T.bucket[P.nchunks]) return;
  const int c = csr_bucket_chunk(P, T, u);
  const int64_t bucket = u - T.bucket[c];
  const uint32_t tot = P.totals[u];
  const uint32_t e0 = P.bucket_start[u + c];
  uint32_t it = P.item_start[u + c];
  int4* items = P.items + T.item[c];
  const uint32_t per = static_cast<uint32_t>(P.tq) * static_cast<uint32_t>(P.item_tiles);
  for (uint32_t off = 0; off < tot; off += per, ++it)
    items[it] = make_int4(static_cast<int>(bucket), static_cast<int>(e0 + off), static_cast<int>(min(per, tot - off)), 0);
}

}  // namespace msa
