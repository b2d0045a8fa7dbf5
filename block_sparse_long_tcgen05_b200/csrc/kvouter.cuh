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
//   m = rowmax(S) * scale * log2e;  P = exp2(S * scale * log2e - m)  (causal mask only where b
//       is the query's own block), written back over S in TMEM as bf16;  l = rowsum(P)
//   O = P V_b            tcgen05.mma, M = 128, N = d, K = 128 keys (TMEM x SMEM) -> TMEM
//   the unnormalised O (bf16) and (m, l) go to the query's slot s; a later pass merges
//   the k slots of every query (no atomics).
//
// Roles (16 warps):
//   warp 0        TMA loads of K_b and V_b
//   warp 1        tcgen05.mma issue (a ready PV goes before the next S)
//   warp 2        TMA gather of query rows (one 2 KB box per 8 rows: both 64-column panels)
//   warp 3        TMA stores of the staged partials
//   warps 4..7    softmax warpgroup 0 (tiles with even index)
//   warps 8..11   softmax warpgroup 1 (odd tiles): the two alternate on the exp unit
//   warps 12..15  epilogue warpgroup: O from TMEM to bf16 staging, for every tile
// Tile n uses TMEM pair w = n % 2 (S/P at column 128*w, O at 256 + 128*w) and staging w.
//
// Shared-memory layouts (all 128-byte swizzled, 1024-byte aligned):
//   K, V: [panel][128 keys][128 B]                     (8-row group stride 1 KB, panel 16 KB)
//   Q, staging: [8-row group][panel][8 rows][128 B]    (8-row group stride kPanels KB, panel 1 KB)
#pragma once
#include "ptx.cuh"

namespace msa {

constexpr int kKvItemTiles = 8;
constexpr int kKvThreads = 512;
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
  float2* ml;                // [chunk rows][G][k][R]: (row max in log2 units, row sum)
};

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
  uint64_t* s_full = bars + 4 + 2 * QS;     // [2] S of tile n in TMEM (MMA -> softmax)
  uint64_t* p_full = s_full + 2;            // [2] P written over S (softmax, 4 warps -> MMA)
  uint64_t* o_full = s_full + 4;            // [2] PV done (MMA -> epilogue; also frees S/P)
  uint64_t* o_free = s_full + 6;            // [2] O read out (epilogue, 4 warps -> MMA)
  uint64_t* stg_full = s_full + 8;          // [2] staging written (epilogue, 4 warps -> store warp)
  uint64_t* stg_empty = s_full + 10;        // [2] staging read by its TMA stores (store warp -> epilogue)
  uint64_t* mma_done = s_full + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1); mbar_init(k_empty, 1); mbar_init(v_full, 1); mbar_init(v_empty, 1);
    for (int i = 0; i < QS; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 4);
      mbar_init(&o_full[i], 1); mbar_init(&o_free[i], 4);
      mbar_init(&stg_full[i], 4); mbar_init(&stg_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
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
  const int4 first_item = (static_cast<int>(blockIdx.x) < n_items) ? P.items[blockIdx.x] : make_int4(0, 0, 0, 0);

  if (warp == 0) {
    // ------------------------------ K / V producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int ni = 0, kn = 0, vn = 0;
      int4 nxt = first_item;
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
    int4 nxt = first_item;
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
    // Event loop over two cursors of this CTA's tile sequence: PV(n) as soon as P(n) is
    // written (it ends warpgroup n%2's cycle), otherwise S(n) as soon as its query rows are
    // loaded and PV(n - 2), which read P from the same TMEM columns, has completed.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, true);
      const uint32_t k_addr = smem_u32(smem + C::kKOff);
      const uint32_t v_addr = smem_u32(smem + C::kVOff);
      struct Cursor {
        int t, j, ntiles, n, ni;
      };
      auto start = [&](Cursor& c) {
        c.t = blockIdx.x; c.j = 0; c.n = 0; c.ni = 0;
        c.ntiles = (c.t < n_items) ? (first_item.z + TQ - 1) / TQ : 0;
      };
      auto advance = [&](Cursor& c) {
        ++c.n;
        if (++c.j == c.ntiles) {
          c.j = 0;
          c.t += grid;
          ++c.ni;
          c.ntiles = (c.t < n_items) ? (__ldg(&P.items[c.t].z) + TQ - 1) / TQ : 0;
        }
      };
      Cursor cs, cp;   // next S to issue, next PV to issue
      start(cs);
      start(cp);
      uint64_t idle_since = 0;
      bool ok = true;
      while (ok && (cs.t < n_items || cp.n < cs.n)) {
        bool progressed = false;
        if (cp.n < cs.n) {
          const int w = cp.n & 1;
          const uint32_t u = static_cast<uint32_t>(cp.n >> 1);
          if ((cp.j != 0 || mbar_test(v_full, cp.ni & 1)) && mbar_test(&p_full[w], u & 1) &&
              mbar_test(&o_free[w], (u & 1) ^ 1)) {
            tc_fence_after();
            const uint32_t d_o = tmem + 256 + w * 128;
            const uint32_t a_p = tmem + w * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_bf16_ts(d_o, a_p + kk * 8, smem_desc(v_addr + kk * 2048, 16384, 1024, kLayoutSw128), idesc_o,
                           kk > 0);
            umma_commit(&o_full[w]);
            if (cp.j == cp.ntiles - 1) umma_commit(v_empty);
            advance(cp);
            progressed = true;
          }
        }
        if (!progressed && cs.t < n_items) {
          const int qs = cs.n % QS;
          const int w = cs.n & 1;
          const uint32_t u = static_cast<uint32_t>(cs.n >> 1);
          if ((cs.j != 0 || mbar_test(k_full, cs.ni & 1)) &&
              mbar_test(&q_full[qs], static_cast<uint32_t>(cs.n / QS) & 1) &&
              mbar_test(&o_full[w], (u & 1) ^ 1)) {
            tc_fence_after();
            const uint32_t q_addr = smem_u32(smem + C::kQOff + qs * C::kTileBytes);
            const uint32_t d_s = tmem + w * 128;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t adesc =
                  smem_desc(q_addr + (kk >> 2) * 1024 + (kk & 3) * 32, 16, C::kGroupBytes, kLayoutSw128);
              const uint64_t bdesc = smem_desc(k_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSw128);
              umma_bf16(d_s, adesc, bdesc, idesc_s, kk > 0);
            }
            umma_commit(&q_empty[qs]);
            umma_commit(&s_full[w]);
            if (cs.j == cs.ntiles - 1) umma_commit(k_empty);
            advance(cs);
            progressed = true;
          }
        }
        if (progressed) {
          idle_since = 0;
        } else {
          // bounded idling: give up (and make every role give up) after the wait limit
          const uint64_t now = globaltimer_ns();
          if (idle_since == 0) idle_since = now;
          if (*abort_flag) ok = false;
          else if (now - idle_since > kWaitLimitNs) {
            record_error(MSA_ERR_TIMEOUT, kKidKvOuter);
            *abort_flag = 1;
            ok = false;
          }
          __nanosleep(20);
        }
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, kKidKvOuter);
    }
  } else if (warp == 3) {
    // ------------------------------ partial stores ------------------------------
    // Once the epilogue warps have staged a tile, lane q issues query q's TMA stores; when
    // every store has read the staging buffer, it is handed back.
    if (lane == 0) tma_prefetch_desc(&tm_o);
    int nt = 0;
    bool ok = true;
    int4 nxt = first_item;
    for (int t = blockIdx.x; t < n_items && ok; t += grid) {
      const int4 it = nxt;
      if (t + grid < n_items) nxt = P.items[t + grid];
      const int g = it.x / P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        const int w = nt & 1;
        const uint32_t u = static_cast<uint32_t>(nt >> 1);
        const int nq = min(TQ, it.z - j * TQ);
        const int e = (lane < nq) ? __ldg(P.entries + it.y + j * TQ + lane) : 0;
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait(&stg_full[w], u & 1, abort_flag, kKidKvOuter) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        if (lane < nq) {
          const int64_t il = static_cast<int64_t>(e >> 5) - P.row0;
          const int row = static_cast<int>((il * P.G + g) * P.k + (e & 31));
          const uint8_t* src = smem + C::kOOff + w * C::kTileBytes + lane * (RP / 8) * C::kGroupBytes;
          if (P.R >= 8) {
#pragma unroll
            for (int h8 = 0; h8 < RP / 8; ++h8) tma_store_4d(&tm_o, src + h8 * C::kGroupBytes, 0, h8 * 8, 0, row);
          } else {
#pragma unroll
            for (int p = 0; p < C::kPanels; ++p) tma_store_4d(&tm_o, src + p * 1024, 0, 0, p, row);
          }
          bulk_commit_group();
          bulk_wait_read_all();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&stg_empty[w]);
      }
    }
    bulk_wait_all();
  } else if (warp >= 12) {
    // ------------------------------ epilogue warpgroup ------------------------------
    // O of every tile: TMEM -> bf16 -> swizzled staging, then handed to the store warp.
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int nt = 0;
    bool fail = false;
    int4 nxt = first_item;
    for (int t = blockIdx.x; t < n_items && !fail; t += grid) {
      const int4 it = nxt;
      if (t + grid < n_items) nxt = P.items[t + grid];
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        const int w = nt & 1;
        const uint32_t u = static_cast<uint32_t>(nt >> 1);
        const uint32_t t_o = tmem + lane_base + 256 + w * 128;
        const uint32_t o_row = smem_u32(smem + C::kOOff + w * C::kTileBytes) + (m >> 3) * C::kGroupBytes + (m & 7) * 128;
        if (!mbar_wait(&o_full[w], u & 1, abort_flag, kKidKvOuter)) { fail = true; break; }
        if (!mbar_wait(&stg_empty[w], (u & 1) ^ 1, abort_flag, kKidKvOuter)) { fail = true; break; }
        tc_fence_after();
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
              const uint32_t* s8 = v[h] + x * 8;
              st_shared_v4(addr, pack_bf16x2(__uint_as_float(s8[0]), __uint_as_float(s8[1])),
                           pack_bf16x2(__uint_as_float(s8[2]), __uint_as_float(s8[3])),
                           pack_bf16x2(__uint_as_float(s8[4]), __uint_as_float(s8[5])),
                           pack_bf16x2(__uint_as_float(s8[6]), __uint_as_float(s8[7])));
            }
          }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&o_free[w]);
          mbar_arrive(&stg_full[w]);
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------ softmax warpgroups ------------------------------
    // The four warps of a warpgroup never wait for one another: each hands its rows over
    // through mbarrier arrivals (P to the MMA warp).
    const int wg = (warp - 4) >> 2;               // 0 or 1: takes tiles with nt % 2 == wg
    const int quad = warp & 3;
    const int m = quad * 32 + lane;               // row of the tile == TMEM lane
    const int q = m / RP, r = m % RP;
    const uint32_t t_s = tmem + (static_cast<uint32_t>(quad * 32) << 16) + wg * 128;
    int nt = 0;
    bool fail = false;
    int e_pref = 0, pref_nt = -1;   // CSR entry of this thread's row in the warpgroup's next tile
    int4 nxt = first_item;
    for (int t = blockIdx.x; t < n_items && !fail; t += grid) {
      const int4 it = nxt;
      if (t + grid < n_items) nxt = P.items[t + grid];
      const int g = it.x / P.nbk, b = it.x % P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        if ((nt & 1) != wg) continue;
        const uint32_t u = static_cast<uint32_t>(nt >> 1);
        const int nq = min(TQ, it.z - j * TQ);
        const bool valid = (q < nq) && (r < P.R);
        const int e = (pref_nt == nt) ? e_pref : (valid ? __ldg(P.entries + it.y + j * TQ + q) : 0);
        const int i = valid ? (e >> 5) : 0;
        const int s = valid ? (e & 31) : 0;
        // load the entry for this warpgroup's next tile now (same item or the next one); rows
        // past that tile's queries read a neighbouring entry that is never used
        {
          int jn = j + 2;
          const int32_t* base = nullptr;
          if (jn < ntiles) {
            base = P.entries + it.y;
          } else if (t + grid < n_items && (jn -= ntiles) < (nxt.z + TQ - 1) / TQ) {
            base = P.entries + nxt.y;
          }
          pref_nt = base ? nt + 2 : -1;
          if (base) e_pref = __ldg(base + jn * TQ + q);
        }
        const int limit = !valid ? -1 : ((b == (i >> 7)) ? (i & 127) : 127);   // keys c <= limit are visible
        // warps whose rows all see the whole block skip the per-key mask
        const bool whole = __all_sync(0xffffffffu, limit == 127);
        // ---- row max (pass 1 over S; two 32-column loads per TMEM wait, 4 independent chains)
        if (!mbar_wait(&s_full[wg], u & 1, abort_flag, kKidKvOuter)) { fail = true; break; }
        tc_fence_after();
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
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
              for (int x = 0; x < 32; x += 2)
                mx4[(x >> 1) & 3] = max3f(mx4[(x >> 1) & 3], __uint_as_float(v[h][x]), __uint_as_float(v[h][x + 1]));
            } else {
#pragma unroll
              for (int x = 0; x < 32; x += 2) {
                const int col = (c + h) * 32 + x;
                const float a0 = (col <= limit) ? __uint_as_float(v[h][x]) : -INFINITY;
                const float a1 = (col + 1 <= limit) ? __uint_as_float(v[h][x + 1]) : -INFINITY;
                mx4[(x >> 1) & 3] = max3f(mx4[(x >> 1) & 3], a0, a1);
              }
            }
          }
        }
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        const float mref = (limit >= 0) ? mx * P.scale_log2 : 0.0f;
        // ---- P = exp2(S * scale * log2e - m), written over S as bf16 (pass 2)
        float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(t_s + c * 32, v);
          tmem_ld_wait();
          uint32_t pk[16];
          if (whole) {
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(v[x]), P.scale_log2, -mref));
              const float p1 = ex2_approx(fmaf(__uint_as_float(v[x + 1]), P.scale_log2, -mref));
              l4[(x >> 1) & 3] += p0 + p1;
              pk[x >> 1] = pack_bf16x2(p0, p1);
            }
          } else {
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const int col = c * 32 + x;
              const float p0 = (col <= limit) ? ex2_approx(fmaf(__uint_as_float(v[x]), P.scale_log2, -mref)) : 0.0f;
              const float p1 =
                  (col + 1 <= limit) ? ex2_approx(fmaf(__uint_as_float(v[x + 1]), P.scale_log2, -mref)) : 0.0f;
              l4[(x >> 1) & 3] += p0 + p1;
              pk[x >> 1] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st16(t_s + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[wg]);
        if (valid) {
          const int64_t il = static_cast<int64_t>(i) - P.row0;
          P.ml[((il * P.G + g) * P.k + s) * P.R + r] = make_float2(mref, (l4[0] + l4[1]) + (l4[2] + l4[3]));
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

}  // namespace msa
