// Index-branch KL loss, forward, executed KV-outer.
//
// hyper.ai "MiniMax Sparse Attention", Method (fourth paragraph): a KL divergence aligns the
// Index Branch's distribution with the Main Branch's on the selected tokens; zhichai.net
// section 5.1: the Main Branch side is the group-averaged distribution. For query i and
// group g, over the tokens T of its selected blocks (j <= i):
//   P_main(j) = (1 / R) sum_h exp(l_h(j) - lse_h),   l_h(j) = scale * q[i, h] . k[j, g]
//   P_idx(j)  = exp(c y(j) - LSE_y),                  y(j) = q_idx[i, g] . k_idx[j, g]
//   KL = sum_j P_main(j) (ln P_main(j) - c y(j) + LSE_y)
//      = A - c B + C LSE_y,   A = sum P_main ln P_main,  B = sum P_main y,  C = sum P_main
// with lse_h the Main Branch's log-sum-exp over T (an output of the forward) and LSE_y the
// index scores' log-sum-exp over T. Each (query, slot) contributes the sums over one block;
// a merge adds the slots of a query in ascending order (no atomics).
//
// A work item is (group g, block b, up to kKvItemTiles query tiles) from the same inverted
// index as the KV-outer attention pass; a tile holds TQ = 128 / RP queries, query q owning
// rows [q RP, q RP + R) as there. Per tile, with K_b and K_idx,b in shared memory:
//   S = Q K_b^T       tcgen05.mma, M = 128, N = BK, K = D    -> TMEM region w
//   Y = Qi K_idx,b^T  tcgen05.mma, M = 128, N = BK, K = DI   -> TMEM region 2 + w
// where Qi repeats each query's index row on all of its RP rows, so every thread reads its
// query's y(j) from its own TMEM lane. A thread computes exp(l_h(j) - lse_h) for its row;
// the RP rows of a query (consecutive lanes of one warp) are summed by a reduce-scatter
// over those lanes, after which each lane owns BK / 8 keys of P_main, adds them into A, B
// and C and folds its keys' c y(j) into a running (max, sum); the lanes of the query then
// combine those and one writes the slot's partial (A, B, C, m_y, l_y).
//
// Roles (12 warps):
//   warp 0      TMA loads of K_b and K_idx,b (one buffer each; the next item's block loads
//               once every product of the current item has completed)
//   warp 1      tcgen05.mma issue of S and Y, in tile order
//   warp 2      query gather: TMA boxes of q as in the KV-outer pass; the index rows by
//               16-byte loads, written RP times into the swizzled Qi tile (one query per
//               store instruction, so the lanes' stores fall into distinct banks)
//   warp 3      idle
//   warps 4-11  two reduction warpgroups; tile n goes to warpgroup n % 2
#pragma once
#include <cuda_bf16.h>

#include "kvouter.cuh"

namespace msa {

constexpr int kKlThreads = 12 * 32;
constexpr int kKlQStages = 2;

template <int D, int RP, int BK, int DI>
struct KlCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;               // Q tile
  static constexpr int kGroupBytes = kPanels * 1024;           // one 8-row group of Q, all panels
  static constexpr bool kISw64 = (DI == 32);
  static constexpr int kIRowBytes = kISw64 ? 64 : 128;         // bytes per row per index panel
  static constexpr int kIPanels = kISw64 ? 1 : DI / 64;
  static constexpr int kIAtom = 8 * kIRowBytes;                // one 8-row swizzle atom
  static constexpr int kIGroupBytes = kIPanels * kIAtom;       // one 8-row group of Qi, all panels
  static constexpr int kITileBytes = 128 * DI * 2;             // Qi tile
  static constexpr uint32_t kILayout = kISw64 ? kLayoutSw64 : kLayoutSw128;
  static constexpr int kKBytes = BK * D * 2;
  static constexpr int kKPanel = BK * 128;
  static constexpr int kKiBytes = BK * DI * 2;
  static constexpr int kKiPanel = BK * kIRowBytes;
  static constexpr int TQ = 128 / RP;
  static constexpr int kKOff = 0;
  static constexpr int kKiOff = kKOff + kKBytes;
  static constexpr int kQOff = (kKiOff + kKiBytes + 1023) / 1024 * 1024;
  static constexpr int kQiOff = kQOff + kKlQStages * kTileBytes;
  static constexpr int kBarOff = kQiOff + kKlQStages * kITileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
};

struct KlParams {
  const int32_t* entries;
  const int4* items;
  const uint32_t* n_items;   // device scalar
  const __nv_bfloat16* q_idx;   // [N][G][DI]
  const float* lse;             // [N][Hq]: the Main Branch's log-sum-exp (natural log)
  int G, R, k, nbk;
  int64_t row0;
  float scale_log2;             // scale * log2(e)
  float idx_scale_log2;         // c * log2(e)
  float* part;                  // [chunk rows][G][k][8]: A, B, C, m_y (log2 units), l_y
};

// tensor maps: tm_q as the KV-outer pass; tm_k: k [N][G][D] as (D, G, N), box (64, 1, BK);
// tm_ki: k_idx [N][G][DI] as (DI, G, N), box (kIRowBytes / 2, 1, BK)
template <int D, int RP, int BK, int DI>
__global__ void __launch_bounds__(kKlThreads, 1)
kl_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_ki, const __grid_constant__ KlParams P) {
  using C = KlCfg<D, RP, BK, DI>;
  constexpr int TQ = C::TQ;
  constexpr int QS = kKlQStages;
  constexpr int NCH = BK / 32;
  static_assert(RP == 8, "the reduce-scatter runs over the 8 rows of a query");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;              // [QS]
  uint64_t* q_empty = bars + 2 + QS;        // [QS]
  uint64_t* s_full = bars + 2 + 2 * QS;     // [2] S and Y of tile n in TMEM
  uint64_t* sp_free = s_full + 2;           // [2] the warpgroup has read S and Y
  uint64_t* mma_done = sp_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  WaitCtl* abort_flag = reinterpret_cast<WaitCtl*>(tmem_slot + 2);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < QS; ++i) { mbar_init(&q_full[i], 2); mbar_init(&q_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&s_full[i], 1); mbar_init(&sp_free[i], 4); }
    mbar_init(mma_done, 1);
    wait_ctl_init(abort_flag);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = static_cast<int>(*P.n_items);
  const int grid = static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ------------------------------ K / K_idx producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_ki);
      int ni = 0;
      for (int t = blockIdx.x; t < n_items; t += grid, ++ni) {
        const int4 it = P.items[t];
        const int g = it.x / P.nbk, b = it.x % P.nbk;
        if (!mbar_wait(kv_empty, (ni & 1) ^ 1, abort_flag, kKidKl)) break;
        mbar_arrive_expect_tx(kv_full, C::kKBytes + C::kKiBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(smem + C::kKOff + p * C::kKPanel, &tm_k, kv_full, p * 64, g, b * BK);
        for (int p = 0; p < C::kIPanels; ++p)
          tma_load_3d(smem + C::kKiOff + p * C::kKiPanel, &tm_ki, kv_full, p * (C::kIRowBytes / 2), g, b * BK);
      }
      if (ni > 0) mbar_wait(kv_full, (ni - 1) & 1, nullptr, kKidKl);   // the last loads land before exit
    }
  } else if (warp == 2) {
    // ------------------------------ query gather ------------------------------
    if (lane == 0) tma_prefetch_desc(&tm_q);
    int nt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_items && ok; t += grid) {
      const int4 it = P.items[t];
      const int g = it.x / P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        const int qs = nt % QS;
        const uint32_t qu = static_cast<uint32_t>(nt / QS);
        const int nq = min(TQ, it.z - j * TQ);
        const int e = (lane < nq) ? __ldg(P.entries + it.y + j * TQ + lane) : 0;
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait(&q_empty[qs], (qu & 1) ^ 1, abort_flag, kKidKl) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(&q_full[qs], nq * RP * 128 * C::kPanels);
        __syncwarp();
        if (lane < nq)
          tma_load_4d(smem + C::kQOff + qs * C::kTileBytes + lane * C::kGroupBytes, &tm_q, &q_full[qs], 0, g * P.R, 0,
                      e >> 5);
        {
          // Each query's index row, RP copies (one per row of the query's 8-row group). The whole
          // warp writes one query at a time: lane l takes 16-byte chunk l % CPR of the row into
          // rows (l / CPR) + t * (32 / CPR), so the lanes of one store hit distinct banks.
          constexpr int CPR = DI / 8;                 // 16-byte chunks per row
          constexpr int RPI = 32 / CPR;               // rows written per store instruction
          const int ch = lane % CPR, rsub = lane / CPR;
          const int pnl = (ch * 16) / C::kIRowBytes;
          const int cin = ((ch * 16) % C::kIRowBytes) / 16;
          uint4 row[TQ];                              // chunk ch of every query's row, loads in flight together
#pragma unroll
          for (int qq = 0; qq < TQ; ++qq) {
            const int eq = __shfl_sync(0xffffffffu, e, qq);
            row[qq] = (qq < nq) ? __ldg(reinterpret_cast<const uint4*>(
                                       P.q_idx + (static_cast<int64_t>(eq >> 5) * P.G + g) * DI) + ch)
                                : make_uint4(0u, 0u, 0u, 0u);
          }
          uint8_t* tile = smem + C::kQiOff + qs * C::kITileBytes;
#pragma unroll
          for (int qq = 0; qq < TQ; ++qq) {
            if (qq < nq) {
              uint8_t* grp = tile + qq * C::kIGroupBytes + pnl * C::kIAtom;
#pragma unroll
              for (int t = 0; t < RP / RPI; ++t) {
                const int r = rsub + t * RPI;
                const int sw = C::kISw64 ? (cin ^ ((r >> 1) & 3)) : (cin ^ r);
                st_shared_v4(smem_u32(grp + r * C::kIRowBytes + sw * 16), row[qq].x, row[qq].y, row[qq].z, row[qq].w);
              }
            }
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_full[qs]);
      }
    }
    if (lane == 0) {
      for (int b2 = 0; b2 < QS; ++b2) {
        if (nt > b2) {
          const int last = ((nt - 1 - b2) / QS) * QS + b2;
          mbar_wait(&q_full[b2], static_cast<uint32_t>(last / QS) & 1, nullptr, kKidKl);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BK, false);
      const uint32_t k_addr = smem_u32(smem + C::kKOff);
      const uint32_t ki_addr = smem_u32(smem + C::kKiOff);
      int n = 0, ni = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_items && ok; t += grid, ++ni) {
        const int4 it = P.items[t];
        const int ntiles = (it.z + TQ - 1) / TQ;
        if (!mbar_wait(kv_full, ni & 1, abort_flag, kKidKl)) { ok = false; break; }
        for (int j = 0; j < ntiles; ++j, ++n) {
          const int w = n & 1;
          const uint32_t u = static_cast<uint32_t>(n >> 1) & 1;
          const int qs = n % QS;
          if (!mbar_wait(&q_full[qs], static_cast<uint32_t>(n / QS) & 1, abort_flag, kKidKl) ||
              !mbar_wait(&sp_free[w], u ^ 1, abort_flag, kKidKl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(smem + C::kQOff + qs * C::kTileBytes);
          const uint32_t qi_addr = smem_u32(smem + C::kQiOff + qs * C::kITileBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t adesc = smem_desc(q_addr + (kk >> 2) * 1024 + (kk & 3) * 32, 16, C::kGroupBytes, kLayoutSw128);
            const uint64_t bdesc = smem_desc(k_addr + (kk >> 2) * C::kKPanel + (kk & 3) * 32, 16, 1024, kLayoutSw128);
            umma_bf16(tmem + w * 128, adesc, bdesc, idesc, kk > 0);
          }
          constexpr int KPR = C::kIRowBytes / 32;    // K-steps per index panel row
#pragma unroll
          for (int kk = 0; kk < DI / 16; ++kk) {
            const uint32_t off_a = (kk / KPR) * C::kIAtom + (kk % KPR) * 32;
            const uint32_t off_b = (kk / KPR) * C::kKiPanel + (kk % KPR) * 32;
            const uint64_t adesc = smem_desc(qi_addr + off_a, 16, C::kIGroupBytes, C::kILayout);
            const uint64_t bdesc = smem_desc(ki_addr + off_b, 16, C::kIAtom, C::kILayout);
            umma_bf16(tmem + 256 + w * 128, adesc, bdesc, idesc, kk > 0);
          }
          umma_commit(&q_empty[qs]);
          umma_commit(&s_full[w]);
          if (j == ntiles - 1) umma_commit(kv_empty);
        }
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, kKidKl);
    }
  } else if (warp >= 4) {
    // ------------------------------ reduction warpgroups ------------------------------
    const int wg = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int m = quad * 32 + lane;               // row of the tile == TMEM lane
    const int q = m / RP, r = m % RP;
    const uint32_t t_s = tmem + (static_cast<uint32_t>(quad * 32) << 16) + wg * 128;
    const uint32_t t_y = t_s + 256;
    const int Hq = P.G * P.R;
    int nt = 0;
    bool fail = false;
    for (int t = blockIdx.x; t < n_items && !fail; t += grid) {
      const int4 it = P.items[t];
      const int g = it.x / P.nbk, b = it.x % P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        if ((nt & 1) != wg) continue;
        const uint32_t u = static_cast<uint32_t>(nt >> 1) & 1;
        const int nq = min(TQ, it.z - j * TQ);
        const bool qvalid = q < nq;
        const bool valid = qvalid && (r < P.R);
        const int e = qvalid ? __ldg(P.entries + it.y + j * TQ + q) : 0;
        const int i = e >> 5, s = e & 31;
        const int limit = !qvalid ? -1 : ((b == i / BK) ? (i % BK) : BK - 1);   // keys c <= limit are visible
        const float lse2 = valid ? __ldg(P.lse + static_cast<int64_t>(i) * Hq + g * P.R + r) * 1.4426950408889634f : 0.0f;
        if (!mbar_wait(&s_full[wg], u, abort_flag, kKidKl)) { fail = true; break; }
        tc_fence_after();
        float A = 0.0f, Bsum = 0.0f, Csum = 0.0f, my = -INFINITY, ly = 0.0f;
        const int b2 = (r >> 2) & 1, b1 = (r >> 1) & 1, b0 = r & 1;
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {
          uint32_t vs[32], vy[32];
          tmem_ld32(t_s + c * 32, vs);
          tmem_ld32(t_y + c * 32, vy);
          tmem_ld_wait();
          if (c == NCH - 1) {   // S and Y of this tile fully read: hand the TMEM region back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sp_free[wg]);
          }
          float p[32], y[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const int col = c * 32 + x;
            p[x] = (valid && col <= limit) ? ex2_approx(fmaf(__uint_as_float(vs[x]), P.scale_log2, -lse2)) : 0.0f;
            y[x] = __uint_as_float(vy[x]);
          }
          // reduce-scatter of p over the 8 lanes of the query; y follows the same selection
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float keep = b2 ? p[x + 16] : p[x], give = b2 ? p[x] : p[x + 16];
            p[x] = keep + __shfl_xor_sync(0xffffffffu, give, 4);
            y[x] = b2 ? y[x + 16] : y[x];
          }
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float keep = b1 ? p[x + 8] : p[x], give = b1 ? p[x] : p[x + 8];
            p[x] = keep + __shfl_xor_sync(0xffffffffu, give, 2);
            y[x] = b1 ? y[x + 8] : y[x];
          }
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float keep = b0 ? p[x + 4] : p[x], give = b0 ? p[x] : p[x + 4];
            p[x] = keep + __shfl_xor_sync(0xffffffffu, give, 1);
            y[x] = b0 ? y[x + 4] : y[x];
          }
          // this lane's 4 keys: columns c * 32 + 16 b2 + 8 b1 + 4 b0 + x
          const float inv_r = 1.0f / static_cast<float>(P.R);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int col = c * 32 + 16 * b2 + 8 * b1 + 4 * b0 + x;
            const float pm = p[x] * inv_r;
            if (pm > 0.0f) A = fmaf(pm, __log2f(pm) * 0.6931471805599453f, A);
            Bsum = fmaf(pm, y[x], Bsum);
            Csum += pm;
            if (col <= limit) {
              const float y2 = y[x] * P.idx_scale_log2;
              const float mn = fmaxf(my, y2);
              ly = ly * ex2_approx(my - mn) + ex2_approx(y2 - mn);
              my = mn;
            }
          }
        }
        // combine the 8 lanes of the query
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          A += __shfl_xor_sync(0xffffffffu, A, o);
          Bsum += __shfl_xor_sync(0xffffffffu, Bsum, o);
          Csum += __shfl_xor_sync(0xffffffffu, Csum, o);
          const float mo = __shfl_xor_sync(0xffffffffu, my, o);
          const float lo = __shfl_xor_sync(0xffffffffu, ly, o);
          const float mn = fmaxf(my, mo);
          ly = (mn == -INFINITY) ? 0.0f : ly * ex2_approx(my - mn) + lo * ex2_approx(mo - mn);
          my = mn;
        }
        if (qvalid && r == 0) {
          const int64_t il = static_cast<int64_t>(i) - P.row0;
          float* dst = P.part + ((il * P.G + g) * P.k + s) * 8;
          reinterpret_cast<float4*>(dst)[0] = make_float4(A, Bsum, Csum, my);
          reinterpret_cast<float4*>(dst)[1] = make_float4(ly, 0.0f, 0.0f, 0.0f);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

struct KlMergeParams {
  const float* part;          // [rows][G][k][8]
  const int32_t* block_ids;   // [N][G][k]
  float* kl;                  // [N][G]
  int64_t row0, rows;
  int G, k;
  float idx_scale;
};

// one thread per (query, group): the valid slots in ascending order, then
// KL = A - c B + C LSE_y (natural log units)
__global__ void __launch_bounds__(256) kl_merge_kernel(const __grid_constant__ KlMergeParams P) {
  const int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (u >= P.rows * P.G) return;
  const int64_t i = P.row0 + u / P.G;
  const int g = static_cast<int>(u % P.G);
  const int32_t* ids = P.block_ids + (i * P.G + g) * P.k;
  const float* part = P.part + u * P.k * 8;
  float A = 0.0f, B = 0.0f, Cs = 0.0f, M = -INFINITY;
  for (int s = 0; s < P.k; ++s) {
    if (ids[s] < 0) break;
    A += part[s * 8 + 0];
    B += part[s * 8 + 1];
    Cs += part[s * 8 + 2];
    M = fmaxf(M, part[s * 8 + 3]);
  }
  float L = 0.0f;
  for (int s = 0; s < P.k; ++s) {
    if (ids[s] < 0) break;
    L += part[s * 8 + 4] * exp2f(part[s * 8 + 3] - M);
  }
  const float lse = (M + log2f(L)) * 0.6931471805599453f;
  P.kl[i * P.G + g] = A - P.idx_scale * B + Cs * lse;
}

}  // namespace msa
