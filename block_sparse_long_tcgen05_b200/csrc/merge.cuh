// Log-sum-exp merge of per-slot partials (prefill chunks and decode).
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
  float* lse;                  // optional [rows0 + rows][Hq]: log-sum-exp of the logits (natural log)
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
// Six groups: the consumers' latency sets the pass's rate (two groups measured 17% slower
// than three, six 1.5-2% faster than three at 128K).
#ifndef MSA_MERGE_GROUPS
#define MSA_MERGE_GROUPS 6
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

// kLse: also write each (query, head)'s log-sum-exp (a separate instantiation, so the common
// path carries no code for it).
template <int D, bool kLse>
__global__ void __launch_bounds__(kMergeThreads, 1)
merge_stream_kernel(const __grid_constant__ MergeParams P, const __grid_constant__ MergeStreamLayout S) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S.stages * S.stage_bytes);
  uint64_t* empty = full + S.stages;
  WaitCtl* abort_flag = reinterpret_cast<WaitCtl*>(empty + S.stages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S.stages; ++s) {
      mbar_init(&full[s], 1 + 32);          // expect_tx arrival + one arrival per producer lane
      mbar_init(&empty[s], kMergeGroupThreads / 32);   // the four warps of the unit's group
    }
    wait_ctl_init(abort_flag);
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
          if constexpr (kLse) {   // logits are in log2 units: scale back by ln 2
            if (lane == 0) P.lse[(P.row0 + u / P.G) * Hq + (u % P.G) * P.R + r] = (M + __log2f(W)) * 0.6931471805599453f;
          }
        }
      }
      __syncwarp();
      const int64_t i = P.row0 + u / P.G;
      const int g = static_cast<int>(u % P.G);
      // ---- combine: thread task (r, c) = head r, 16-byte chunk c of its D-wide row
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

}  // namespace msa
