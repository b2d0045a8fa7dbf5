// Index Branch, part 2: exp-free Top-k over block maxima, local block forced.
//
// zhichai.net article, section 4.1 "Exp-free Top-K": selection only needs the relative
// order of the index scores, so no exp / softmax is taken; hyper.ai "MiniMax Sparse
// Attention", Method: the Top-K blocks per query group are kept and the local block is
// always included.
//
// Keys are 64-bit: (order-preserving uint32 of the block max) << 32 | (0xFFFFFFFF - kb),
// so a larger key means a higher score, and among equal scores the lower block index.
// Every key is distinct, so the selected set is unique. One thread owns one
// (query, group) row and keeps the best k - 1 keys seen so far in registers, sorted
// descending (insertion on a strict '>' test).
#pragma once
#include "ptx.cuh"

namespace msa {

template <int KM>
__device__ __forceinline__ void topk_insert(uint64_t (&L)[KM], uint64_t key) {
  static_assert(KM >= 1, "at least one non-local place");
  if (key > L[KM - 1]) {
#pragma unroll
    for (int p = KM - 1; p > 0; --p) L[p] = (key > L[p - 1]) ? L[p - 1] : ((key > L[p]) ? key : L[p]);
    L[0] = key > L[0] ? key : L[0];
  }
}

// The same insertion for a caller that offers the blocks in ascending order of kb: 32-bit
// ordered scores with the ids alongside. A block never displaces an equal score already in
// the list (strict comparisons), which is the tie rule (equal scores: the lower block id
// ranks first), because every block already in the list has a lower id.
template <int KM>
__device__ __forceinline__ void topk_insert_ascending(uint32_t (&Ls)[KM], int (&Lb)[KM], uint32_t u, int kb) {
  static_assert(KM >= 1, "at least one non-local place");
  if (u > Ls[KM - 1]) {
#pragma unroll
    for (int p = KM - 1; p > 0; --p) {
      const bool down = u > Ls[p - 1];   // the entry above moves down into place p
      const bool here = u > Ls[p];
      Ls[p] = down ? Ls[p - 1] : (here ? u : Ls[p]);
      Lb[p] = down ? Lb[p - 1] : (here ? kb : Lb[p]);
    }
    if (u > Ls[0]) {
      Ls[0] = u;
      Lb[0] = kb;
    }
  }
}

// Select for one row: src[kb * stride] holds the ordered key of block kb for
// kb in [0, bl); bl is the local block. Writes KM + 1 ids (ascending) to out.
// Requires bl >= KM + 1 (more non-local candidates than places).
template <int KM>
__device__ __forceinline__ void topk_select_row(const uint32_t* __restrict__ src, int64_t stride, int bl,
                                                int32_t* __restrict__ out) {
  if constexpr (KM == 0) {
    out[0] = bl;
    return;
  } else {
  uint64_t L[KM];
#pragma unroll
  for (int p = 0; p < KM; ++p) L[p] = 0ull;   // below every real key (ordered keys are > 0)
  int kb = 0;
  for (; kb + 8 <= bl; kb += 8) {
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(src + static_cast<int64_t>(kb + u) * stride);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      topk_insert<KM>(L, (static_cast<uint64_t>(v[u]) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - (kb + u)));
  }
  for (; kb < bl; ++kb) {
    const uint32_t v = __ldg(src + static_cast<int64_t>(kb) * stride);
    topk_insert<KM>(L, (static_cast<uint64_t>(v) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - kb));
  }
  int ids[KM];
#pragma unroll
  for (int p = 0; p < KM; ++p) ids[p] = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(L[p]));
  // odd-even transposition sort, ascending
#pragma unroll
  for (int pass = 0; pass < KM; ++pass) {
#pragma unroll
    for (int p = pass & 1; p + 1 < KM; p += 2) {
      const int a = ids[p], b = ids[p + 1];
      ids[p] = min(a, b);
      ids[p + 1] = max(a, b);
    }
  }
#pragma unroll
  for (int p = 0; p < KM; ++p) out[p] = ids[p];
  out[KM] = bl;
  }
}

__device__ __forceinline__ void topk_all_visible(int bl, int k, int32_t* __restrict__ out) {
  for (int s = 0; s < k; ++s) out[s] = (s <= bl) ? s : -1;
}

struct TopkPrefillParams {
  const uint32_t* maxima;
  int32_t* block_ids;       // [N, G, k]
  int64_t N;
  int G, k, qb0;
  int64_t region_per_group;
};

// grid (query blocks of the launch, G), 128 threads: thread r owns row qb * 128 + r.
template <int KM>
__global__ void __launch_bounds__(128) topk_prefill_kernel(const __grid_constant__ TopkPrefillParams P) {
  const int qb = P.qb0 + blockIdx.x;
  const int g = blockIdx.y;
  const int r = threadIdx.x;
  const int64_t i = static_cast<int64_t>(qb) * 128 + r;
  if (i >= P.N) return;
  int32_t* out = P.block_ids + (i * P.G + g) * P.k;
  if (qb + 1 <= P.k) {
    topk_all_visible(qb, P.k, out);
    return;
  }
  const int64_t region = 128ll * ((static_cast<int64_t>(qb) * (qb - 1)) / 2 -
                                  (static_cast<int64_t>(P.qb0) * (P.qb0 - 1)) / 2);
  const uint32_t* src = P.maxima + static_cast<int64_t>(g) * P.region_per_group + region + r;
  topk_select_row<KM>(src, 128, qb, out);
}

struct TopkDecodeParams {
  const uint32_t* maxima;   // [B, G, nbmax]
  int32_t* block_ids;       // [B, G, k]
  const int32_t* seqlens;
  int B, G, k, nbmax, bk;
};

}  // namespace msa
