// Main Branch, KV-outer (KV-stationary) execution.
//
// hyper.ai "MiniMax Sparse Attention", Method (third paragraph): exact scaled dot-product
// softmax attention restricted to the tokens of the selected blocks; Key Contributions:
// KV-outer sparse attention keeps tensor cores busy under block-granular access and
// handles skewed block popularity without atomic updates (zhichai.net section 4.2).
//
// A work item is (group g, block b, up to kKvItemTiles tiles of the queries that chose b).
// A tile holds TQ = 128 / RP queries; query q of the tile owns rows [q*RP, q*RP + R) of a
// 128-row operand, RP = max(R, 8), so every query starts on an 8-row group.
// Per tile, with K_b / V_b resident in shared memory:
//   S = Q K_b^T          tcgen05.mma, M = 128 rows, N = 128 keys, K = d (SMEM x SMEM) -> TMEM
//   P = exp2(S * scale * log2e - rowmax)   (causal mask only where b is the query's own block),
//       written back over S in TMEM as bf16
//   O = P V_b            tcgen05.mma, M = 128, N = d, K = 128 keys (TMEM x SMEM) -> TMEM
//   partial (O / rowsum) as bf16 and lse = rowmax + ln(rowsum) go to the query's slot s,
//   and a later pass merges the k slots of every query (no atomics).
//
// Roles (12 warps): warp 0 loads K_b / V_b with TMA, warp 2 gathers query rows with TMA
// (one 2 KB box per 8 rows: both 64-column panels), warp 1 issues the MMAs, and two
// softmax warpgroups (warps 4..7 and 8..11) take alternate tiles, so one runs softmax
// while the other drains its O accumulator and stores partials. Warpgroup w always uses
// TMEM accumulator pair w (S/P at column 128*w, O at 256 + 128*w) and staging buffer w.
//
// Shared-memory layouts (all 128-byte swizzled, 1024-byte aligned):
//   K, V: [panel][128 keys][128 B]                     (8-row group stride 1 KB, panel 16 KB)
//   Q, staging: [8-row group][panel][8 rows][128 B]    (8-row group stride kPanels KB, panel 1 KB)
#pragma once
#include "ptx.cuh"

namespace msa {

constexpr int kKvItemTiles = 8;
constexpr int kKvThreads = 384;
constexpr int kKvQStages = 3;

template <int D, int RP>
struct KvCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kGroupBytes = kPanels * 1024;     // one 8-row group, all panels
  static constexpr int TQ = 128 / RP;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kQOff = 2 * kTileBytes;
  static constexpr int kOOff = kQOff + kKvQStages * kTileBytes;   // 2 staging buffers
  static constexpr int kBarOff = kOOff + 2 * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
};

struct KvParams {
  const int32_t* entries;
  const int4* items;
  const uint32_t* n_items;   // device scalar
  int G, R, k, nbk;
  int64_t row0;              // first query of the chunk
  float scale_log2;
  float* lse;                // [chunk rows][G][k][R]
};

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                             int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16 (A read from tensor memory).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns, store.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// tensor maps:
//   tm_q: 4-D view of q [N][Hq][D] as (64 elems, Hq heads, D/64 panels, N), box (64, 8, D/64, 1)
//   tm_k, tm_v: 3-D view of k / v [N][G][D] as (D, G, N), box (64, 1, 128)
//   tm_o: 4-D view of the partials [rows][R][D] as (64, R, D/64, rows),
//         box (64, min(R, 8), R >= 8 ? D/64 : 1, 1)
template <int D, int RP>
__global__ void __launch_bounds__(kKvThreads, 1)
kvouter_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ KvParams P) {
  using C = KvCfg<D, RP>;
  constexpr int TQ = C::TQ;
  constexpr int QS = kKvQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* k_full = bars + 0;
  uint64_t* k_empty = bars + 1;
  uint64_t* v_full = bars + 2;
  uint64_t* v_empty = bars + 3;
  uint64_t* q_full = bars + 4;              // [QS]
  uint64_t* q_empty = bars + 4 + QS;        // [QS]
  uint64_t* s_full = bars + 4 + 2 * QS;     // [2]
  uint64_t* p_full = s_full + 2;            // [2]
  uint64_t* o_full = s_full + 4;            // [2]
  uint64_t* o_free = s_full + 6;            // [2]
  uint64_t* mma_done = s_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* wg_fail = reinterpret_cast<volatile int*>(tmem_slot + 2);   // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1); mbar_init(k_empty, 1); mbar_init(v_full, 1); mbar_init(v_empty, 1);
    for (int i = 0; i < QS; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 4);
      mbar_init(&o_full[i], 1); mbar_init(&o_free[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    wg_fail[0] = 0;
    wg_fail[1] = 0;
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
    // ------------------------------ K / V producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int ni = 0, kn = 0, vn = 0;
      int4 nxt = (static_cast<int>(blockIdx.x) < n_items) ? P.items[blockIdx.x] : make_int4(0, 0, 0, 0);
      for (int t = blockIdx.x; t < n_items; t += grid, ++ni) {
        const int4 it = nxt;
        if (t + grid < n_items) nxt = P.items[t + grid];
        const int g = it.x / P.nbk, b = it.x % P.nbk;
        if (!mbar_wait(k_empty, (ni & 1) ^ 1, abort_flag, kKidKvOuter)) break;
        mbar_arrive_expect_tx(k_full, C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(smem + C::kKOff + p * 16384, &tm_k, k_full, p * 64, g, b * 128);
        ++kn;
        if (!mbar_wait(v_empty, (ni & 1) ^ 1, abort_flag, kKidKvOuter)) break;
        mbar_arrive_expect_tx(v_full, C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(smem + C::kVOff + p * 16384, &tm_v, v_full, p * 64, g, b * 128);
        ++vn;
      }
      // drain: the last K and V loads issued must land before the CTA exits
      if (kn > 0) mbar_wait(k_full, (kn - 1) & 1, nullptr, kKidKvOuter);
      if (vn > 0) mbar_wait(v_full, (vn - 1) & 1, nullptr, kKidKvOuter);
    }
  } else if (warp == 2) {
    // ------------------------------ query gather ------------------------------
    // Lane q of the warp owns query q of the tile: it loads the CSR entry and issues that
    // query's boxes (RP / 8 boxes of 8 heads x all panels).
    if (lane == 0) tma_prefetch_desc(&tm_q);
    int nt = 0;
    bool ok = true;
    int4 nxt = (static_cast<int>(blockIdx.x) < n_items) ? P.items[blockIdx.x] : make_int4(0, 0, 0, 0);
    for (int t = blockIdx.x; t < n_items && ok; t += grid) {
      const int4 it = nxt;
      if (t + grid < n_items) nxt = P.items[t + grid];
      const int g = it.x / P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        const int qs = nt % QS;
        const uint32_t qu = static_cast<uint32_t>(nt / QS);
        const int nq = min(TQ, it.z - j * TQ);
        const int e = (lane < nq) ? __ldg(P.entries + it.y + j * TQ + lane) : 0;
        int w_ok = 1;   // lane 0 waits; the verdict is broadcast so the warp stays uniform
        if (lane == 0) w_ok = mbar_wait(&q_empty[qs], (qu & 1) ^ 1, abort_flag, kKidKvOuter) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(&q_full[qs], nq * RP * 128 * C::kPanels);
        __syncwarp();
        if (lane < nq) {
          uint8_t* dst = smem + C::kQOff + qs * C::kTileBytes + lane * (RP / 8) * C::kGroupBytes;
#pragma unroll
          for (int h8 = 0; h8 < RP / 8; ++h8)
            tma_load_4d(dst + h8 * C::kGroupBytes, &tm_q, &q_full[qs], 0, g * P.R + h8 * 8, 0, e >> 5);
        }
      }
    }
    if (lane == 0) {
      for (int b2 = 0; b2 < QS; ++b2) {
        if (nt > b2) {
          const int last = ((nt - 1 - b2) / QS) * QS + b2;
          mbar_wait(&q_full[b2], static_cast<uint32_t>(last / QS) & 1, nullptr, kKidKvOuter);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, true);
      const uint32_t k_addr = smem_u32(smem + C::kKOff);
      const uint32_t v_addr = smem_u32(smem + C::kVOff);
      int nt = 0, ni = 0;
      bool ok = true;
      int pd_nt = -1, pd_first = 0, pd_last = 0, pd_ni = 0;   // pending PV
      auto issue_pv = [&](int tnt, int first, int last, int tni) -> bool {
        const int w = tnt & 1;
        const uint32_t u = static_cast<uint32_t>(tnt >> 1);
        if (first && !mbar_wait(v_full, tni & 1, abort_flag, kKidKvOuter)) return false;
        if (!mbar_wait(&p_full[w], u & 1, abort_flag, kKidKvOuter)) return false;
        if (!mbar_wait(&o_free[w], (u & 1) ^ 1, abort_flag, kKidKvOuter)) return false;
        tc_fence_after();
        const uint32_t d_o = tmem + 256 + w * 128;
        const uint32_t a_p = tmem + w * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(d_o, a_p + kk * 8, smem_desc(v_addr + kk * 2048, 16384, 1024, kLayoutSw128), idesc_o,
                       kk > 0);
        umma_commit(&o_full[w]);
        if (last) umma_commit(v_empty);
        return true;
      };
      int4 nxt = (static_cast<int>(blockIdx.x) < n_items) ? P.items[blockIdx.x] : make_int4(0, 0, 0, 0);
      for (int t = blockIdx.x; t < n_items && ok; t += grid, ++ni) {
        const int4 it = nxt;
        if (t + grid < n_items) nxt = P.items[t + grid];
        const int ntiles = (it.z + TQ - 1) / TQ;
        if (!mbar_wait(k_full, ni & 1, abort_flag, kKidKvOuter)) { ok = false; break; }
        for (int j = 0; j < ntiles; ++j, ++nt) {
          const int qs = nt % QS;
          const int w = nt & 1;
          const uint32_t u = static_cast<uint32_t>(nt >> 1);
          if (!mbar_wait(&q_full[qs], static_cast<uint32_t>(nt / QS) & 1, abort_flag, kKidKvOuter)) { ok = false; break; }
          // S/P buffer w is free once PV of tile nt - 2 (which read P from it) completed
          if (!mbar_wait(&o_full[w], (u & 1) ^ 1, abort_flag, kKidKvOuter)) { ok = false; break; }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(smem + C::kQOff + qs * C::kTileBytes);
          const uint32_t d_s = tmem + w * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t adesc = smem_desc(q_addr + (kk >> 2) * 1024 + (kk & 3) * 32, 16, C::kGroupBytes, kLayoutSw128);
            const uint64_t bdesc = smem_desc(k_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSw128);
            umma_bf16(d_s, adesc, bdesc, idesc_s, kk > 0);
          }
          umma_commit(&q_empty[qs]);
          umma_commit(&s_full[w]);
          if (j == ntiles - 1) umma_commit(k_empty);
          if (pd_nt >= 0 && !issue_pv(pd_nt, pd_first, pd_last, pd_ni)) { ok = false; pd_nt = -1; break; }
          pd_nt = nt; pd_first = (j == 0); pd_last = (j == ntiles - 1); pd_ni = ni;
        }
      }
      if (ok && pd_nt >= 0) issue_pv(pd_nt, pd_first, pd_last, pd_ni);
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, kKidKvOuter);
    }
  } else if (warp >= 4) {
    // ------------------------------ softmax warpgroups ------------------------------
    const int wg = (warp - 4) >> 2;               // 0 or 1: takes tiles with nt % 2 == wg
    const int quad = warp & 3;
    const int m = quad * 32 + lane;               // row of the tile == TMEM lane
    const int q = m / RP, r = m % RP;
    const bool storer = (quad == 0);              // lanes of the warpgroup's first warp store
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + wg * 128;
    const uint32_t t_o = tmem + lane_base + 256 + wg * 128;
    uint8_t* o_s = smem + C::kOOff + wg * C::kTileBytes;
    const uint32_t o_row = smem_u32(o_s) + (m >> 3) * C::kGroupBytes + (m & 7) * 128;
    const uint32_t bar_id = 1 + wg;
    int nt = 0;
    bool fail = false, stop = false;
    int4 nxt = (static_cast<int>(blockIdx.x) < n_items) ? P.items[blockIdx.x] : make_int4(0, 0, 0, 0);
    for (int t = blockIdx.x; t < n_items && !stop; t += grid) {
      const int4 it = nxt;
      if (t + grid < n_items) nxt = P.items[t + grid];
      const int g = it.x / P.nbk, b = it.x % P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        if ((nt & 1) != wg) continue;
        const uint32_t u = static_cast<uint32_t>(nt >> 1);
        const int nq = min(TQ, it.z - j * TQ);
        const bool valid = (q < nq) && (r < P.R);
        int i = 0, s = 0;
        if (valid) {
          const int e = __ldg(P.entries + it.y + j * TQ + q);
          i = e >> 5;
          s = e & 31;
        }
        const int e_store = (storer && lane < nq) ? __ldg(P.entries + it.y + j * TQ + lane) : 0;
        // warm L1 with the entries of this warpgroup's next tile (same item or the next one)
        if (lane == 0) {
          const int jn = j + 2;
          const int32_t* pe = (jn < ntiles) ? P.entries + it.y + jn * TQ
                                            : P.entries + nxt.y + (jn - ntiles) * TQ;
          asm volatile("prefetch.global.L1 [%0];" ::"l"(pe));
          asm volatile("prefetch.global.L1 [%0];" ::"l"(pe + TQ - 1));
        }
        const int limit = !valid ? -1 : ((b == (i >> 7)) ? (i & 127) : 127);   // keys c <= limit are visible
        // warps whose rows all see the whole block skip the per-key mask
        const bool whole = __all_sync(0xffffffffu, limit == 127);
        // ---- row max (pass 1 over S; two 32-column loads per TMEM wait)
        if (!fail && !mbar_wait(&s_full[wg], u & 1, abort_flag, kKidKvOuter)) fail = true;
        tc_fence_after();
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          uint32_t v[2][32];
          tmem_ld32(t_s + c * 32, v[0]);
          tmem_ld32(t_s + c * 32 + 32, v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (whole) {
#pragma unroll
              for (int x = 0; x < 32; x += 2) mx = max3f(mx, __uint_as_float(v[h][x]), __uint_as_float(v[h][x + 1]));
            } else {
#pragma unroll
              for (int x = 0; x < 32; x += 2) {
                const int col = (c + h) * 32 + x;
                const float a0 = (col <= limit) ? __uint_as_float(v[h][x]) : -INFINITY;
                const float a1 = (col + 1 <= limit) ? __uint_as_float(v[h][x + 1]) : -INFINITY;
                mx = max3f(mx, a0, a1);
              }
            }
          }
        }
        const float mref = (limit >= 0) ? mx * P.scale_log2 : 0.0f;
        // ---- P = exp2(S * scale * log2e - max), written over S as bf16 (pass 2)
        float l = 0.0f;
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          uint32_t v[2][32];
          tmem_ld32(t_s + c * 32, v[0]);
          tmem_ld32(t_s + c * 32 + 32, v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[16];
            if (whole) {
#pragma unroll
              for (int x = 0; x < 32; x += 2) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(v[h][x]), P.scale_log2, -mref));
                const float p1 = ex2_approx(fmaf(__uint_as_float(v[h][x + 1]), P.scale_log2, -mref));
                l += p0 + p1;
                pk[x >> 1] = pack_bf16x2(p0, p1);
              }
            } else {
#pragma unroll
              for (int x = 0; x < 32; x += 2) {
                const int col = (c + h) * 32 + x;
                const float p0 =
                    (col <= limit) ? ex2_approx(fmaf(__uint_as_float(v[h][x]), P.scale_log2, -mref)) : 0.0f;
                const float p1 =
                    (col + 1 <= limit) ? ex2_approx(fmaf(__uint_as_float(v[h][x + 1]), P.scale_log2, -mref)) : 0.0f;
                l += p0 + p1;
                pk[x >> 1] = pack_bf16x2(p0, p1);
              }
            }
            tmem_st16(t_s + (c + h) * 16, pk);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[wg]);
        // ---- O -> registers, normalise, stage
        if (!fail && !mbar_wait(&o_full[wg], u & 1, abort_flag, kKidKvOuter)) fail = true;
        tc_fence_after();
        const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
        if (storer) bulk_wait_read_all();            // this buffer's previous stores have read it
        named_bar_sync(bar_id, 128);
#pragma unroll 1
        for (int c = 0; c < D / 32; c += 2) {
          uint32_t v[2][32];
          tmem_ld32(t_o + c * 32, v[0]);
          tmem_ld32(t_o + c * 32 + 32, v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {              // four 16-byte chunks of 8 columns
              const int ch = (c + h) * 4 + x;          // chunk index along d
              const uint32_t addr = o_row + (ch >> 3) * 1024 + (((ch & 7) ^ (m & 7)) << 4);
              const uint32_t* w = v[h] + x * 8;
              st_shared_v4(addr, pack_bf16x2(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv),
                           pack_bf16x2(__uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv),
                           pack_bf16x2(__uint_as_float(w[4]) * inv, __uint_as_float(w[5]) * inv),
                           pack_bf16x2(__uint_as_float(w[6]) * inv, __uint_as_float(w[7]) * inv));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[wg]);
        if (valid) {
          const int64_t il = static_cast<int64_t>(i) - P.row0;
          P.lse[((il * P.G + g) * P.k + s) * P.R + r] = (mref + __log2f(l)) * 0.69314718055994531f;
        }
        fence_proxy_async_smem();
        if (fail) wg_fail[wg] = 1;
        named_bar_sync(bar_id, 128);
        if (storer && lane < nq) {   // lane q stores query q
          const int64_t il = static_cast<int64_t>(e_store >> 5) - P.row0;
          const int row = static_cast<int>((il * P.G + g) * P.k + (e_store & 31));
          const uint8_t* src = o_s + lane * (RP / 8) * C::kGroupBytes;
          if (P.R >= 8) {
#pragma unroll
            for (int h8 = 0; h8 < RP / 8; ++h8) tma_store_4d(&tm_o, src + h8 * C::kGroupBytes, 0, h8 * 8, 0, row);
          } else {
#pragma unroll
            for (int p = 0; p < C::kPanels; ++p) tma_store_4d(&tm_o, src + p * 1024, 0, 0, p, row);
          }
          bulk_commit_group();
        }
        // uniform stop decision for the warpgroup (flag written before the barrier above)
        stop = wg_fail[wg] != 0;
        if (stop) break;
      }
    }
    if (storer) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace msa
