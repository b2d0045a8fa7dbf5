// Query-stationary decode kernels: Index Branch scan of one new query per sequence and the
// sparse attention over its selected blocks (merged by merge_kernel).
#pragma once
#include <cuda_bf16.h>

#include "merge.cuh"
#include "ptx.cuh"
#include "topk.cuh"

namespace msa {

// ------------------------------------------------------------------------------------
// Decode, Index Branch: block maxima of the one new query per sequence against every
// full block before its local block (query-stationary: the index-key cache streams
// through once, 64 contiguous bytes per lane per load). Blocks hold bk in {32, 64, 128}
// tokens; a CTA scans 128 tokens, i.e. 128 / bk blocks.
// ------------------------------------------------------------------------------------
struct DecodeScanParams {
  const __nv_bfloat16* q_idx;   // [B][G][DI]
  const __nv_bfloat16* k_idx;   // [B][Lmax][G][DI]
  const int32_t* seqlens;
  uint32_t* maxima;             // [B][G][nbmax]
  int B, G, nbmax, bk;
  int64_t Lmax;
};

// grid (ceil(Lmax / 128), B), 256 threads: one CTA per (sequence, 128-token span). Needs
// G * DI / 32 to be a power of two <= 32 (checked by the host).
template <int DI>
__global__ void __launch_bounds__(256) decode_scan_kernel(const __grid_constant__ DecodeScanParams P) {
  __shared__ uint32_t smax[128];   // [G][4]
  const int b = blockIdx.y, kb = blockIdx.x;
  const int L = P.seqlens[b];
  if (L < 1 || L > P.Lmax) {
    if (kb == 0 && threadIdx.x == 0) record_error(MSA_ERR_DEVICE_BOUNDS, kKidDecodeScan);
    return;
  }
  const int bl = (L - 1) / P.bk;                    // local block: only blocks before it are scanned
  const int ntok = min(128, bl * P.bk - kb * 128);  // tokens of this span in those blocks
  if (ntok <= 0) return;
  const int cpt = P.G * DI / 32;             // 64-byte chunks per token
  constexpr int LPG = DI / 32;               // lanes (chunks) per group
  const int lane = threadIdx.x & 31;
  const int w = lane % cpt;                  // constant per lane since cpt | 32
  const int g = w / LPG;
  const int qoff = (w % LPG) * 32;
  if (threadIdx.x < 128) smax[threadIdx.x] = 0u;
  float qv[32];
  {
    const uint4* qp = reinterpret_cast<const uint4*>(P.q_idx + (static_cast<int64_t>(b) * P.G + g) * DI + qoff);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 raw = __ldg(qp + u);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(h2[t]);
        qv[u * 8 + 2 * t] = f.x;
        qv[u * 8 + 2 * t + 1] = f.y;
      }
    }
  }
  __syncthreads();
  const uint4* base = reinterpret_cast<const uint4*>(P.k_idx + (static_cast<int64_t>(b) * P.Lmax + kb * 128) *
                                                                   P.G * DI);
  const int nchunks = ntok * cpt;
  float best[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // per block of the span
  for (int c0 = threadIdx.x; c0 < nchunks; c0 += 256 * 2) {
    uint4 raw[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = c0 + h * 256;
#pragma unroll
      for (int u = 0; u < 4; ++u) raw[h][u] = (c < nchunks) ? __ldg(base + static_cast<int64_t>(c) * 4 + u) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float acc = 0.0f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[h][u]);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = __bfloat1622float2(h2[t]);
          acc = fmaf(qv[u * 8 + 2 * t], f.x, acc);
          acc = fmaf(qv[u * 8 + 2 * t + 1], f.y, acc);
        }
      }
#pragma unroll
      for (int o = 1; o < LPG; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int c = c0 + h * 256;
      const int f = (c / cpt) / P.bk;   // block of the span holding this token
#pragma unroll
      for (int ff = 0; ff < 4; ++ff)
        if (c < nchunks && ff == f) best[ff] = fmaxf(best[ff], acc);
    }
  }
  if ((lane % LPG) == 0) {
#pragma unroll
    for (int ff = 0; ff < 4; ++ff) {
      if (best[ff] == -INFINITY) continue;   // no token of that block in this lane's share
      float m = __fadd_rn(best[ff], 0.0f);
      uint32_t u = __float_as_uint(m);
      u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
      atomicMax(&smax[g * 4 + ff], u);
    }
  }
  __syncthreads();
  const int F = 128 / P.bk;
  for (int e = threadIdx.x; e < P.G * F; e += blockDim.x) {
    const int gg = e / F, ff = e % F;
    const int blk = kb * F + ff;
    if (blk < bl) P.maxima[(static_cast<int64_t>(b) * P.G + gg) * P.nbmax + blk] = smax[gg * 4 + ff];
  }
}

// ------------------------------------------------------------------------------------
// Decode, Main Branch: one CTA per (sequence, group, slot): exact softmax attention of
// the group's R heads over the slot's block (causal in the local block), written as an
// unnormalised partial with its (row max, row sum) for the merge kernel.
// ------------------------------------------------------------------------------------
// Decode Top-k over the scanned block maxima [B][G][nbmax].
// One warp per (sequence, group) row. Lane l keeps the running top list of blocks
// l, l + 32, l + 64, ... (ascending, so the 32-bit insertion keeps the tie rule); the 32 lane
// lists are then merged in KM rounds, each taking the warp's best head by the full key
// (score, then lower block id) and advancing the winning lane's list.
template <int KM>
__global__ void __launch_bounds__(256) topk_decode_kernel(const __grid_constant__ TopkDecodeParams P) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= P.B * P.G) return;
  const int b = row / P.G;
  const int L = P.seqlens[b];
  int32_t* out = P.block_ids + static_cast<int64_t>(row) * P.k;
  if (L < 1 || (L - 1) / P.bk >= P.nbmax) {  // host validated lmax; guard anyway
    if (lane == 0) record_error(MSA_ERR_DEVICE_BOUNDS, kKidTopk);
    for (int s = lane; s < P.k; s += 32) out[s] = -1;
    return;
  }
  const int bl = (L - 1) / P.bk;
  if (bl + 1 <= P.k) {
    if (lane == 0) topk_all_visible(bl, P.k, out);
    return;
  }
  if constexpr (KM == 0) {   // k = 1: the local block alone
    if (lane == 0) out[0] = bl;
  } else {
  const uint32_t* src = P.maxima + static_cast<int64_t>(row) * P.nbmax;
  uint32_t Ls[KM];
  int Lb[KM];
#pragma unroll
  for (int p = 0; p < KM; ++p) { Ls[p] = 0u; Lb[p] = -1; }
  for (int kb = lane; kb < bl; kb += 32) topk_insert_ascending<KM>(Ls, Lb, __ldg(src + kb), kb);
  int ids[KM];
#pragma unroll
  for (int r = 0; r < KM; ++r) {
    // this lane's head as a 64-bit key (0 when its list is exhausted: below every real key)
    uint64_t key = (Lb[0] >= 0) ? ((static_cast<uint64_t>(Ls[0]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(Lb[0])))
                                : 0ull;
    uint64_t best = key;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    ids[r] = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best));
    if (key == best) {   // keys are unique (distinct block ids): exactly one lane advances
#pragma unroll
      for (int p = 0; p + 1 < KM; ++p) { Ls[p] = Ls[p + 1]; Lb[p] = Lb[p + 1]; }
      Ls[KM - 1] = 0u;
      Lb[KM - 1] = -1;
    }
  }
  // odd-even transposition sort, ascending (the same on every lane)
#pragma unroll
  for (int pass = 0; pass < KM; ++pass) {
#pragma unroll
    for (int p = pass & 1; p + 1 < KM; p += 2) {
      const int a = ids[p], c = ids[p + 1];
      ids[p] = min(a, c);
      ids[p + 1] = max(a, c);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int p = 0; p < KM; ++p) out[p] = ids[p];
    out[KM] = bl;
  }
  }
}

// 16-byte asynchronous global -> shared copy (bypassing L1); with ok == false nothing is
// read and the 16 shared bytes are zero-filled. Both addresses 16-byte aligned.
__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(sdst)), "l"(gsrc), "r"(ok ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

struct DecodeAttnParams {
  const __nv_bfloat16* q;       // [B][Hq][D]
  const __nv_bfloat16* kc;      // [B][Lmax][G][D]
  const __nv_bfloat16* vc;
  const int32_t* seqlens;
  const int32_t* block_ids;     // [B][G][k]
  __nv_bfloat16* opart;         // [B][G][k][R][D]
  float2* ml;                   // [B][G][k][R]
  int B, G, R, k, bk;
  int64_t Lmax;
  float scale_log2;
};

// Warp-level tensor-core helpers (mma.sync m16n8k16, bf16 in, fp32 accumulate). The decode
// products have M = R <= 16 query heads, too few rows for tcgen05 (M >= 64).
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t (&r)[2], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One CTA (4 warps) per (sequence, group, slot): K / V of the selected block staged in shared
// memory, S = Q K^T and O = P V on tensor cores (M = 16 rows: the group's R <= 16 heads, the
// rest zero), the softmax per head in between. Fragment coordinates: lane = 4 * gq + tq.
template <int D>
__global__ void __launch_bounds__(128) decode_attn_kernel(const __grid_constant__ DecodeAttnParams P) {
  constexpr int KS = D + 8;    // padded smem row: the 8 rows of an ldmatrix hit distinct banks
  extern __shared__ uint8_t dsm[];
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(dsm);
  __nv_bfloat16* Vs = Ks + 128 * KS;
  float* Ss = reinterpret_cast<float*>(Vs + 128 * KS);   // [R][128]: scores, then P
  float* stat = Ss + P.R * 128;                          // [R][2]: max, sum
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int blk = P.block_ids[(static_cast<int64_t>(b) * P.G + g) * P.k + s];
  if (blk < 0) return;
  const int L = P.seqlens[b];
  const int pos = L - 1;
  if (L < 1 || L > P.Lmax || blk > pos / P.bk) {
    if (threadIdx.x == 0) record_error(MSA_ERR_DEVICE_BOUNDS, kKidDecodeAttn);
    return;
  }
  const int j0 = blk * P.bk;
  const int nvalid = min(P.bk, pos - j0 + 1);   // rows past it (beyond the block or the query) stay zero
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  // K / V rows of the block, 16-byte asynchronous copies all in flight at once (rows past
  // the query are zero-filled: source size 0)
  constexpr int CPR = D / 8;
  for (int e = tid; e < 128 * CPR; e += 128) {
    const int j = e / CPR, c = e % CPR;
    const bool ok = j < nvalid;
    const int64_t off = ok ? ((static_cast<int64_t>(b) * P.Lmax + j0 + j) * P.G + g) * D + c * 8 : 0;
    cp_async16(Ks + j * KS + c * 8, P.kc + off, ok);
    cp_async16(Vs + j * KS + c * 8, P.vc + off, ok);
  }
  const __nv_bfloat16* q0 = P.q + (static_cast<int64_t>(b) * P.G * P.R + g * P.R) * D;   // head 0 of the group
  const bool r_lo = gq < P.R, r_hi = gq + 8 < P.R;
  auto qpair = [&](int r, int col) -> uint32_t { return *reinterpret_cast<const uint32_t*>(q0 + r * D + col); };
  cp_async_wait_all();
  __syncthreads();
  // ---- S = Q K^T: warp w takes keys [32 w, 32 w + 32) as four 8-key tiles
  {
    float acc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[nt][x] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int k0 = kk * 16;
      uint32_t a[4];
      a[0] = r_lo ? qpair(gq, k0 + 2 * tq) : 0u;
      a[1] = r_hi ? qpair(gq + 8, k0 + 2 * tq) : 0u;
      a[2] = r_lo ? qpair(gq, k0 + 8 + 2 * tq) : 0u;
      a[3] = r_hi ? qpair(gq + 8, k0 + 8 + 2 * tq) : 0u;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int n0 = warp * 32 + nt * 8;
        uint32_t bf[2];   // keys n0 .. n0 + 7; dims k0 .. k0 + 7 (matrix 0) and k0 + 8 .. (matrix 1)
        ldsm_x2(bf, Ks + (n0 + (lane & 7)) * KS + k0 + 8 * ((lane >> 3) & 1));
        mma_16816(acc[nt], a, bf);
      }
    }
    // scores in log2 units; keys past the query -> -inf
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int n = warp * 32 + nt * 8 + 2 * tq;
      if (r_lo) {
        Ss[gq * 128 + n] = (n < nvalid) ? acc[nt][0] * P.scale_log2 : -INFINITY;
        Ss[gq * 128 + n + 1] = (n + 1 < nvalid) ? acc[nt][1] * P.scale_log2 : -INFINITY;
      }
      if (r_hi) {
        Ss[(gq + 8) * 128 + n] = (n < nvalid) ? acc[nt][2] * P.scale_log2 : -INFINITY;
        Ss[(gq + 8) * 128 + n + 1] = (n + 1 < nvalid) ? acc[nt][3] * P.scale_log2 : -INFINITY;
      }
    }
  }
  __syncthreads();
  // softmax per head: warp w takes heads w, w + 4, ...; P = 2^(x - max) overwrites the scores
  for (int r = warp; r < P.R; r += 4) {
    float v4[4];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < 4; ++u) { v4[u] = Ss[r * 128 + lane + 32 * u]; mx = fmaxf(mx, v4[u]); }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
#pragma unroll
    for (int u = 0; u < 4; ++u) { v4[u] = exp2f(v4[u] - mx); sum += v4[u]; Ss[r * 128 + lane + 32 * u] = v4[u]; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) { stat[2 * r] = mx; stat[2 * r + 1] = sum; }
  }
  __syncthreads();
  const int64_t slot = (static_cast<int64_t>(b) * P.G + g) * P.k + s;
  // ---- O = P V (P as bf16): warp w takes dims [w D / 4, (w + 1) D / 4) as D / 32 tiles of 8
  {
    constexpr int NT = D / 32;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[nt][x] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int k0 = kk * 16;
      uint32_t a[4];
      a[0] = r_lo ? pack_bf16x2(Ss[gq * 128 + k0 + 2 * tq], Ss[gq * 128 + k0 + 2 * tq + 1]) : 0u;
      a[1] = r_hi ? pack_bf16x2(Ss[(gq + 8) * 128 + k0 + 2 * tq], Ss[(gq + 8) * 128 + k0 + 2 * tq + 1]) : 0u;
      a[2] = r_lo ? pack_bf16x2(Ss[gq * 128 + k0 + 8 + 2 * tq], Ss[gq * 128 + k0 + 9 + 2 * tq]) : 0u;
      a[3] = r_hi ? pack_bf16x2(Ss[(gq + 8) * 128 + k0 + 8 + 2 * tq], Ss[(gq + 8) * 128 + k0 + 9 + 2 * tq]) : 0u;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n0 = warp * (D / 4) + nt * 8;
        uint32_t bf[2];   // keys k0 .. k0 + 7 (matrix 0) and k0 + 8 .. k0 + 15 (matrix 1), dims n0 .. n0 + 7
        ldsm_x2_trans(bf, Vs + (k0 + (lane & 15)) * KS + n0);
        mma_16816(acc[nt], a, bf);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = warp * (D / 4) + nt * 8 + 2 * tq;
      if (r_lo)
        *reinterpret_cast<uint32_t*>(P.opart + (slot * P.R + gq) * D + n) = pack_bf16x2(acc[nt][0], acc[nt][1]);
      if (r_hi)
        *reinterpret_cast<uint32_t*>(P.opart + (slot * P.R + gq + 8) * D + n) = pack_bf16x2(acc[nt][2], acc[nt][3]);
    }
  }
  if (tid < P.R) P.ml[slot * P.R + tid] = make_float2(stat[2 * tid], stat[2 * tid + 1]);
}

}  // namespace msa
