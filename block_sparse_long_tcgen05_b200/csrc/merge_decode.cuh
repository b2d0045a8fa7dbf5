// Log-sum-exp merge of per-slot partials, and the query-stationary decode kernels.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace msa {

// ------------------------------------------------------------------------------------
// Merge. Slot s of (query i, group g) holds, per head, the unnormalised partial
// O_s = sum_j 2^(x_j - m_s) v_j over the tokens of one selected block (x_j the logits in
// log2 units), its row max m_s and row sum l_s = sum_j 2^(x_j - m_s). With M = max_s m_s
// and w_s = 2^(m_s - M):
//     o[i, h] = sum_s w_s O_s / sum_s w_s l_s,
// which is exactly the softmax over the union of the selected blocks. Valid slots are
// combined in ascending slot order (a fixed-order fp32 reduction; no atomics).
// ------------------------------------------------------------------------------------
struct MergeParams {
  const __nv_bfloat16* opart;  // [rows][G][k][R][D]
  const float2* ml;            // [rows][G][k][R]: (m_s, l_s)
  const int32_t* block_ids;    // [rows0 + rows][G][k] (absolute row index)
  __nv_bfloat16* o;            // [rows0 + rows][Hq][D]
  int64_t row0, rows;
  int G, R, k;
};

template <int D>
__global__ void __launch_bounds__(256, 2) merge_kernel(const __grid_constant__ MergeParams P) {
  constexpr int LPH = D / 8;          // lanes per head row (16 bytes each)
  constexpr int HPW = 32 / LPH;       // head rows per warp
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t hh = gw * HPW + lane / LPH;
  const int c = lane % LPH;
  if (hh >= P.rows * P.G * P.R) return;
  const int r = static_cast<int>(hh % P.R);
  const int g = static_cast<int>((hh / P.R) % P.G);
  const int64_t il = hh / (static_cast<int64_t>(P.R) * P.G);
  const int64_t i = P.row0 + il;
  const int32_t* ids = P.block_ids + (i * P.G + g) * P.k;
  const int64_t slot0 = (il * P.G + g) * P.k;
  const uint4* prow = reinterpret_cast<const uint4*>(P.opart + (slot0 * P.R + r) * D) + c;
  const int64_t pstride = static_cast<int64_t>(P.R) * D / 8;   // uint4 per slot
  // The LPH lanes of this head row own slots c, c + LPH, ... for ids and (m, l). Every load
  // of the row (ids, (m, l) and the partials of the first 16 slots) is issued before any is
  // used, so a row costs one memory round trip; slots past the valid ones are loaded but
  // never used (they hold no partial).
  const unsigned gmask = (LPH == 32) ? 0xffffffffu : (((1u << LPH) - 1u) << (lane & ~(LPH - 1)));
  const int lane0 = lane & ~(LPH - 1);
  int idv[4];
  float own[4], lsum[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int s = c + LPH * j;
    idv[j] = (s < P.k) ? __ldg(ids + s) : -1;
    const float2 ml = (s < P.k) ? __ldg(P.ml + (slot0 + s) * P.R + r) : make_float2(-INFINITY, 0.0f);
    own[j] = ml.x;
    lsum[j] = ml.y;
  }
  uint4 raw[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) raw[u] = (u < P.k) ? __ldg(prow + u * pstride) : make_uint4(0, 0, 0, 0);
  int nv = 0;   // valid ids come first (ascending, -1 padded)
#pragma unroll
  for (int j = 0; j < 4; ++j) nv += __popc(__ballot_sync(gmask, idv[j] >= 0) & gmask);
#pragma unroll
  for (int j = 0; j < 4; ++j) own[j] = (c + LPH * j < nv) ? own[j] : -INFINITY;
  float M = fmaxf(fmaxf(own[0], own[1]), fmaxf(own[2], own[3]));
#pragma unroll
  for (int o = 1; o < LPH; o <<= 1) M = fmaxf(M, __shfl_xor_sync(gmask, M, o));
#pragma unroll
  for (int j = 0; j < 4; ++j) own[j] = (c + LPH * j < nv) ? ex2_approx(own[j] - M) : 0.0f;
  float acc[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
  float W = 0.0f;
  auto accumulate = [&](const uint4& rw, int s) {   // ascending slot order
    const int j = s / LPH;
    const float mine = (j == 0) ? own[0] : (j == 1) ? own[1] : (j == 2) ? own[2] : own[3];
    const float myl = (j == 0) ? lsum[0] : (j == 1) ? lsum[1] : (j == 2) ? lsum[2] : lsum[3];
    const float wu = __shfl_sync(gmask, mine, lane0 + (s % LPH));
    const float lu = __shfl_sync(gmask, myl, lane0 + (s % LPH));
    if (s < nv) {
      W = fmaf(wu, lu, W);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&rw);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(h2[t]);
        acc[2 * t] = fmaf(wu, f.x, acc[2 * t]);
        acc[2 * t + 1] = fmaf(wu, f.y, acc[2 * t + 1]);
      }
    }
  };
#pragma unroll
  for (int u = 0; u < 16; ++u) accumulate(raw[u], u);
#pragma unroll 1
  for (int s = 16; s < P.k; ++s) {   // k > 16: the remaining slots one by one (uniform trip count)
    const uint4 rw = (s < nv) ? __ldg(prow + s * pstride) : make_uint4(0, 0, 0, 0);
    accumulate(rw, s);
  }
  const float inv = (W > 0.0f) ? 1.0f / W : 0.0f;
  uint4 out;
  out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  out.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  out.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  const int Hq = P.G * P.R;
  reinterpret_cast<uint4*>(P.o + (i * Hq + g * P.R + r) * D)[c] = out;
}

// ------------------------------------------------------------------------------------
// Streaming variant of the merge for the prefill chunks. One unit = one (query, group): its
// k * R * D * 2-byte slab of partials is contiguous, so a producer warp brings it, with the
// unit's (m, l) pairs and block ids, into a ring of shared-memory stages by bulk copy.
// kMergeGroups consumer groups of four warps take units in turn. Per unit each warp first
// turns the (m, l) pairs of the heads it combines into normalised weights
// w_s = 2^(m_s - M) / sum_t 2^(m_t - M) l_t (one lane per slot), written next to the slab;
// then every thread combines one 16-byte chunk of one head row over the valid slots in
// ascending order. Enough groups and stages stay in flight per SM for the pass to run at
// HBM bandwidth on a fraction of the SMs.
// ------------------------------------------------------------------------------------
#ifndef MSA_MERGE_GROUPS
#define MSA_MERGE_GROUPS 3
#endif
constexpr int kMergeGroups = MSA_MERGE_GROUPS;   // consumer groups compiled in (S.groups of them run)
constexpr int kMergeGroupThreads = 128;
constexpr int kMergeThreads = 32 + kMergeGroups * kMergeGroupThreads;

struct MergeStreamLayout {
  int slab_bytes;   // k * R * D * 2
  int ml_off;       // offset of the (m, l) pairs inside a stage
  int ids_off;      // offset of the block ids
  int w_off;        // offset of the weights (k * R floats, written by the consumers)
  int stage_bytes;  // multiple of 128
  int stages;       // a multiple of groups: unit n takes stage n % stages and group n % groups, so
                    // every use of a stage is by the same group, in order (mbarrier parity stays
                    // within one phase)
  int groups;       // active consumer groups, 1 .. kMergeGroups
  int bulk_meta;    // (m, l) and ids rows are 16-byte multiples: copy them in bulk too
};

// bf16 pair (low half first) to two floats: a bf16 is the top half of the float it rounds
__device__ __forceinline__ float bf16lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

template <int D>
__global__ void __launch_bounds__(kMergeThreads, 1)
merge_stream_kernel(const __grid_constant__ MergeParams P, const __grid_constant__ MergeStreamLayout S) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S.stages * S.stage_bytes);
  uint64_t* empty = full + S.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + S.stages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S.stages; ++s) {
      mbar_init(&full[s], 1 + 32);          // expect_tx arrival + one arrival per producer lane
      mbar_init(&empty[s], kMergeGroupThreads / 32);   // the four warps of the unit's group
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int64_t units = P.rows * P.G;
  const int64_t grid = gridDim.x;
  const int kR = P.k * P.R;
  if (warp == 0) {
    // ---- producer: slab by bulk copy, (m, l) and ids by bulk copy or plain loads
    int n = 0;
    for (int64_t u = blockIdx.x; u < units; u += grid, ++n) {
      const int s = n % S.stages;
      const uint32_t ph = static_cast<uint32_t>(n / S.stages);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&empty[s], (ph & 1) ^ 1, abort_flag, kKidMerge) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      uint8_t* st = smem + s * S.stage_bytes;
      const int64_t il = u / P.G, g = u % P.G;
      const float2* mlsrc = P.ml + u * kR;
      const int32_t* idsrc = P.block_ids + ((P.row0 + il) * P.G + g) * P.k;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], S.slab_bytes + (S.bulk_meta ? kR * 8 + P.k * 4 : 0));
        bulk_load_g2s(st, P.opart + u * static_cast<int64_t>(kR) * D, S.slab_bytes, &full[s]);
        if (S.bulk_meta) {
          bulk_load_g2s(st + S.ml_off, mlsrc, kR * 8, &full[s]);
          bulk_load_g2s(st + S.ids_off, idsrc, P.k * 4, &full[s]);
        }
      }
      if (!S.bulk_meta) {
        float2* mldst = reinterpret_cast<float2*>(st + S.ml_off);
        for (int e = lane; e < kR; e += 32) mldst[e] = __ldg(mlsrc + e);
        int32_t* iddst = reinterpret_cast<int32_t*>(st + S.ids_off);
        for (int e = lane; e < P.k; e += 32) iddst[e] = __ldg(idsrc + e);
      }
      mbar_arrive(&full[s]);   // each lane: its stores above (if any) are released with this arrival
    }
    if (lane == 0 && n > 0) {   // drain the copies this warp issued
      for (int s = 0; s < S.stages && s < n; ++s) {
        const int last = ((n - 1 - s) / S.stages) * S.stages + s;
        mbar_wait(&full[s], static_cast<uint32_t>(last / S.stages) & 1, nullptr, kKidMerge);
      }
    }
  } else {
    const int ct = threadIdx.x - 32;
    const int grp = ct / kMergeGroupThreads;
    const int gt = ct % kMergeGroupThreads;
    const int gw = gt >> 5;                       // warp within the group
    constexpr int CPR = D / 8;                    // 16-byte chunks per head row
    const int tasks = P.R * CPR;
    const int Hq = P.G * P.R;
    int n = 0;
    for (int64_t u = blockIdx.x; u < units; u += grid, ++n) {
      if (n % S.groups != grp) continue;
      const int s = n % S.stages;
      const uint32_t ph = static_cast<uint32_t>(n / S.stages);
      if (!mbar_wait(&full[s], ph & 1, abort_flag, kKidMerge)) break;
      uint8_t* st = smem + s * S.stage_bytes;
      const float2* ml = reinterpret_cast<const float2*>(st + S.ml_off);
      const int32_t* ids = reinterpret_cast<const int32_t*>(st + S.ids_off);
      float* wt = reinterpret_cast<float*>(st + S.w_off);
      // valid ids come first (ascending, -1 padded); k <= 32, one lane per slot
      const int nv = __popc(__ballot_sync(0xffffffffu, lane < P.k && ids[lane] >= 0));
      // ---- weights of the heads this warp combines (32 is a multiple of CPR, so each head's
      // tasks belong to one warp and no other warp reads its weights)
      for (int t0 = gw * 32; t0 < tasks; t0 += kMergeGroupThreads) {
        const int r_end = min(P.R, (t0 + 32 + CPR - 1) / CPR);
        for (int r = t0 / CPR; r < r_end; ++r) {
          const float2 v = (lane < nv) ? ml[lane * P.R + r] : make_float2(-INFINITY, 0.0f);
          float M = v.x;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
          const float e = (lane < nv) ? ex2_approx(v.x - M) : 0.0f;
          float W = e * v.y;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
          if (lane < P.k) wt[lane * P.R + r] = (W > 0.0f) ? __fdividef(e, W) : 0.0f;
        }
      }
      __syncwarp();
      // ---- combine: thread task (r, c) = head r, 16-byte chunk c of its D-wide row
      const int64_t i = P.row0 + u / P.G;
      const int g = static_cast<int>(u % P.G);
      for (int task = gt; task < tasks; task += kMergeGroupThreads) {
        const int r = task / CPR, c = task % CPR;
        const uint8_t* src = st + (r * D + c * 8) * 2;
        const int rstride = P.R * D * 2;          // bytes from one slot's row to the next
        float acc[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] = 0.0f;
        for (int s0 = 0; s0 < nv; s0 += 4) {      // 4 slots' loads in flight, combined in order
          uint4 raw[4];
          float w[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int sl = s0 + x;
            const bool ok = sl < nv;
            raw[x] = ok ? *reinterpret_cast<const uint4*>(src + sl * rstride) : make_uint4(0, 0, 0, 0);
            w[x] = ok ? wt[sl * P.R + r] : 0.0f;
          }
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            acc[0] = fmaf(w[x], bf16lo(raw[x].x), acc[0]);
            acc[1] = fmaf(w[x], bf16hi(raw[x].x), acc[1]);
            acc[2] = fmaf(w[x], bf16lo(raw[x].y), acc[2]);
            acc[3] = fmaf(w[x], bf16hi(raw[x].y), acc[3]);
            acc[4] = fmaf(w[x], bf16lo(raw[x].z), acc[4]);
            acc[5] = fmaf(w[x], bf16hi(raw[x].z), acc[5]);
            acc[6] = fmaf(w[x], bf16lo(raw[x].w), acc[6]);
            acc[7] = fmaf(w[x], bf16hi(raw[x].w), acc[7]);
          }
        }
        uint4 out;
        out.x = pack_bf16x2(acc[0], acc[1]);
        out.y = pack_bf16x2(acc[2], acc[3]);
        out.z = pack_bf16x2(acc[4], acc[5]);
        out.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4*>(P.o + (i * Hq + g * P.R + r) * D)[c] = out;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
}

// ------------------------------------------------------------------------------------
// Decode, Index Branch: block maxima of the one new query per sequence against every
// full block before its local block (query-stationary: the index-key cache streams
// through once, 64 contiguous bytes per lane per load).
// ------------------------------------------------------------------------------------
struct DecodeScanParams {
  const __nv_bfloat16* q_idx;   // [B][G][DI]
  const __nv_bfloat16* k_idx;   // [B][Lmax][G][DI]
  const int32_t* seqlens;
  uint32_t* maxima;             // [B][G][nbmax]
  int B, G, nbmax;
  int64_t Lmax;
};

// grid (nbmax, B), 256 threads: one CTA per (sequence, block). Needs G * DI / 32 to be
// a power of two <= 32 (checked by the host).
template <int DI>
__global__ void __launch_bounds__(256) decode_scan_kernel(const __grid_constant__ DecodeScanParams P) {
  __shared__ uint32_t smax[32];
  const int b = blockIdx.y, kb = blockIdx.x;
  const int L = P.seqlens[b];
  if (L < 1 || L > P.Lmax) {
    if (kb == 0 && threadIdx.x == 0) record_error(MSA_ERR_DEVICE_BOUNDS, kKidDecodeScan);
    return;
  }
  const int bl = (L - 1) / 128;
  if (kb >= bl) return;
  const int cpt = P.G * DI / 32;             // 64-byte chunks per token
  constexpr int LPG = DI / 32;               // lanes (chunks) per group
  const int lane = threadIdx.x & 31;
  const int w = lane % cpt;                  // constant per lane since cpt | 32
  const int g = w / LPG;
  const int qoff = (w % LPG) * 32;
  if (threadIdx.x < 32) smax[threadIdx.x] = 0u;
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
  const int nchunks = 128 * cpt;
  float best = -INFINITY;
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
      if (c0 + h * 256 < nchunks) best = fmaxf(best, acc);
    }
  }
  if ((lane % LPG) == 0) {
    float m = __fadd_rn(best, 0.0f);
    uint32_t u = __float_as_uint(m);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    atomicMax(&smax[g], u);
  }
  __syncthreads();
  if (threadIdx.x < P.G) P.maxima[(static_cast<int64_t>(b) * P.G + threadIdx.x) * P.nbmax + kb] = smax[threadIdx.x];
}

// ------------------------------------------------------------------------------------
// Decode, Main Branch: one CTA per (sequence, group, slot): exact softmax attention of
// the group's R heads over the slot's block (causal in the local block), written as an
// unnormalised partial with its (row max, row sum) for the merge kernel.
// ------------------------------------------------------------------------------------
struct DecodeAttnParams {
  const __nv_bfloat16* q;       // [B][Hq][D]
  const __nv_bfloat16* kc;      // [B][Lmax][G][D]
  const __nv_bfloat16* vc;
  const int32_t* seqlens;
  const int32_t* block_ids;     // [B][G][k]
  __nv_bfloat16* opart;         // [B][G][k][R][D]
  float2* ml;                   // [B][G][k][R]
  int B, G, R, k;
  int64_t Lmax;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(128) decode_attn_kernel(const __grid_constant__ DecodeAttnParams P) {
  constexpr int KS = D + 8;    // padded smem row (bank spread)
  extern __shared__ uint8_t dsm[];
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(dsm);
  __nv_bfloat16* Vs = Ks + 128 * KS;
  float* Qs = reinterpret_cast<float*>(Vs + 128 * KS);   // [R][D]
  float* Ss = Qs + P.R * D;                              // [R][128]
  float* stat = Ss + P.R * 128;                          // [R][2]: max, 1/sum
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int blk = P.block_ids[(static_cast<int64_t>(b) * P.G + g) * P.k + s];
  if (blk < 0) return;
  const int L = P.seqlens[b];
  const int pos = L - 1;
  if (L < 1 || L > P.Lmax || blk > pos / 128) {
    if (threadIdx.x == 0) record_error(MSA_ERR_DEVICE_BOUNDS, kKidDecodeAttn);
    return;
  }
  const int j0 = blk * 128;
  const int nvalid = min(128, pos - j0 + 1);
  const int tid = threadIdx.x;
  // q rows, pre-scaled into log2 units
  for (int e = tid; e < P.R * D; e += 128) {
    const int r = e / D, dd = e % D;
    Qs[e] = __bfloat162float(P.q[(static_cast<int64_t>(b) * P.G * P.R + g * P.R + r) * D + dd]) * P.scale_log2;
  }
  // K / V rows of the block (16-byte chunks)
  constexpr int CPR = D / 8;
  for (int e = tid; e < 128 * CPR; e += 128) {
    const int j = e / CPR, c = e % CPR;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (j < nvalid) {
      const int64_t off = ((static_cast<int64_t>(b) * P.Lmax + j0 + j) * P.G + g) * D;
      kv = __ldg(reinterpret_cast<const uint4*>(P.kc + off) + c);
      vv = __ldg(reinterpret_cast<const uint4*>(P.vc + off) + c);
    }
    *reinterpret_cast<uint4*>(Ks + j * KS + c * 8) = kv;
    *reinterpret_cast<uint4*>(Vs + j * KS + c * 8) = vv;
  }
  __syncthreads();
  // scores: thread = key
  {
    const int j = tid;
    for (int r = 0; r < P.R; ++r) {
      float acc = 0.0f;
      if (j < nvalid) {
#pragma unroll 4
        for (int c = 0; c < CPR; ++c) {
          const uint4 raw = *reinterpret_cast<const uint4*>(Ks + j * KS + c * 8);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 f = __bfloat1622float2(h2[t]);
            acc = fmaf(Qs[r * D + c * 8 + 2 * t], f.x, acc);
            acc = fmaf(Qs[r * D + c * 8 + 2 * t + 1], f.y, acc);
          }
        }
      }
      Ss[r * 128 + j] = (j < nvalid) ? acc : -INFINITY;
    }
  }
  __syncthreads();
  // softmax per head: warp w takes heads w, w + 4, ...
  {
    const int w = tid >> 5, lane = tid & 31;
    for (int r = w; r < P.R; r += 4) {
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
  }
  __syncthreads();
  const int64_t slot = (static_cast<int64_t>(b) * P.G + g) * P.k + s;
  for (int e = tid; e < P.R * D; e += 128) {
    const int r = e / D, dd = e % D;
    float acc = 0.0f;
    for (int j = 0; j < nvalid; ++j) acc = fmaf(Ss[r * 128 + j], __bfloat162float(Vs[j * KS + dd]), acc);
    P.opart[(slot * P.R + r) * D + dd] = __float2bfloat16_rn(acc);
  }
  if (tid < P.R) P.ml[slot * P.R + tid] = make_float2(stat[2 * tid], stat[2 * tid + 1]);
}

}  // namespace msa
