// Main Branch, KV-outer (KV-stationary) execution.
//
// hyper.ai "MiniMax Sparse Attention", Method (third paragraph): exact scaled dot-product
// softmax attention restricted to the tokens of the selected blocks; Key Contributions:
// KV-outer sparse attention keeps tensor cores busy under block-granular access and
// handles skewed block popularity without atomic updates (zhichai.net section 4.2).
//
// A work item is (group g, block b, up to kKvItemTiles tiles of the queries that chose b);
// blocks hold BK in {32, 64, 128} keys.
// A tile holds TQ = 128 / RP queries; query q of the tile owns rows [q*RP, q*RP + R) of a
// 128-row operand, RP = max(R, 8), so every query starts on an 8-row group.
// Per tile, with K_b / V_b resident in shared memory:
//   S = Q K_b^T          tcgen05.mma, M = 128 rows, N = BK keys, K = d (SMEM x SMEM) -> TMEM
//   m = rowmax(S) * scale * log2e;  P = exp2(S * scale * log2e - m)  (causal mask only where b
//       is the query's own block), written back over S in TMEM as bf16;  l = rowsum(P)
//   O = P V_b            tcgen05.mma, M = 128, N = d, K = BK keys (TMEM x SMEM) -> TMEM
//   the unnormalised O (bf16) and (m, l) go to the query's slot s; a later pass merges
//   the k slots of every query (no atomics).
//
// Roles (16 warps):
//   warp 0        TMA loads of K_b and V_b into a ring of three block slots (K of item i,
//                 V of item i, K of item i + 1, ...): a slot is refilled once the product
//                 that read its previous block has completed
//   warp 1        tcgen05.mma issue of S = Q K^T, in tile order
//   warp 2        TMA gather of query rows (one 2 KB box per 8 rows: both 64-column panels)
//   warp 3        tcgen05.mma issue of O = P V, in tile order. Two issuers, because an issue
//                 sequence stalls while the tensor pipe is busy: a PV that is ready does not
//                 wait behind the S product of the next tile, nor the other way round.
//   softmax       two warpgroups (warps 4-11); tile n goes to warpgroup n % 2 and to TMEM
//                 S/P region n % 3. With three regions for two warpgroups, S(n + 2) needs
//                 only PV(n - 1) to be done, so it is computed while the warpgroup still
//                 works on tile n, and the warpgroup goes from one tile to its next
//                 without waiting for its own PV and S products.
//   epilogue      warps 12-15: O from TMEM to bf16 staging, TMA-stored per query
// TMEM: S/P regions at columns 0, 128 and 256; O (one buffer: the epilogue reads it out
// while the next tile's softmax runs) at column 384.
//
// Shared-memory layouts (all 128-byte swizzled, 1024-byte aligned):
//   K, V: [panel][BK keys][128 B]                      (8-row group stride 1 KB, panel BK * 128 B)
//   Q, O staging: [8-row group][panel][8 rows][128 B]  (8-row group stride kPanels KB, panel 1 KB)
#pragma once
#include "ptx.cuh"

namespace msa {

constexpr int kKvItemTiles = 4;
constexpr int kKvQStages = 3;      // query tiles in shared memory
constexpr int kKvSlots = 3;        // K / V block slots in shared memory
constexpr int kKvSoftmaxWGs = 2;   // softmax warpgroups; tile n goes to n % 2
constexpr int kKvSRegions = 3;     // S/P regions of TMEM (128 columns each); tile n uses n % 3
constexpr int kKvOCol = kKvSRegions * 128;   // the O accumulator (128 columns)
static_assert(kKvOCol + 128 <= 512, "TMEM holds 512 columns");
constexpr int kKvEpiWarp = 4 + 4 * kKvSoftmaxWGs;   // first warp of the epilogue warpgroup
constexpr int kKvThreads = 32 * (kKvEpiWarp + 4);

template <int D, int RP, int BK>
struct KvCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;         // a query (or staging) tile: 128 rows
  static constexpr int kKvBytes = BK * D * 2;            // a K or V block
  static constexpr int kKvPanel = BK * 128;              // one 64-column panel of a K or V block
  static constexpr int kGroupBytes = kPanels * 1024;     // one 8-row group, all panels
  static constexpr int TQ = 128 / RP;
  static constexpr int kKvOff = 0;                       // kKvSlots K / V block slots
  static constexpr int kQOff = kKvSlots * kKvBytes;      // kKvQStages query stages
  static constexpr int kStgOff = kQOff + kKvQStages * kTileBytes;   // O staging (one tile)
  static constexpr int kBarOff = kStgOff + kTileBytes;
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
//   tm_k, tm_v: 3-D view of k / v [N][G][D] as (D, G, N), box (64, 1, BK)
//   tm_o: 4-D view of the partials [rows][R][D] as (64, R, D/64, rows),
//         box (64, min(R, 8), R >= 8 ? D/64 : 1, 1)
template <int D, int RP, int BK>
__global__ void __launch_bounds__(kKvThreads, 1)
kvouter_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ KvParams P) {
  using C = KvCfg<D, RP, BK>;
  static_assert(BK == 32 || BK == 64 || BK == 128, "block size");
  constexpr int NCH = BK / 32;               // 32-column chunks of S per row
  constexpr int TQ = C::TQ;
  constexpr int QS = kKvQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  constexpr int NS = kKvSRegions, NW = kKvSoftmaxWGs, KS = kKvSlots;
  // a slot's loads alternate between K and V blocks, read by different issuers; each issuer
  // waits on its own full barrier, so that it sees every phase of it
  uint64_t* k_full = bars + 0;              // [KS] K block landed in slot s (producer -> S issuer)
  uint64_t* v_full = k_full + KS;           // [KS] V block landed in slot s (producer -> PV issuer)
  uint64_t* kv_empty = v_full + KS;         // [KS] slot s read out (either issuer -> producer)
  uint64_t* q_full = kv_empty + KS;         // [QS]
  uint64_t* q_empty = q_full + QS;          // [QS]
  uint64_t* s_full = q_empty + QS;          // [NS] S of tile n in TMEM (S issuer -> softmax)
  uint64_t* p_full = s_full + NS;           // [NS] P written over S (softmax, 4 warps -> PV issuer)
  uint64_t* sp_free = p_full + NS;          // [NS] PV done: S/P region free (PV issuer -> S issuer)
  uint64_t* o_full = sp_free + NS;          // PV done (PV issuer -> epilogue)
  uint64_t* o_free = o_full + 1;            // O read out (epilogue, 4 warps -> PV issuer)
  uint64_t* s_done = o_free + 1;            // all S products of the CTA complete
  uint64_t* pv_done = s_done + 1;           // all PV products of the CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 1);
  WaitCtl* abort_flag = reinterpret_cast<WaitCtl*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < KS; ++i) { mbar_init(&k_full[i], 1); mbar_init(&v_full[i], 1); mbar_init(&kv_empty[i], 1); }
    for (int i = 0; i < QS; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1); }
    for (int i = 0; i < NS; ++i) { mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 4); mbar_init(&sp_free[i], 1); }
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    mbar_init(s_done, 1);
    mbar_init(pv_done, 1);
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
  const int4 first_item = (static_cast<int>(blockIdx.x) < n_items) ? P.items[blockIdx.x] : make_int4(0, 0, 0, 0);

  if (warp == 0) {
    // ------------------------------ K / V producer ------------------------------
    // Load j (K of item i is j = 2i, its V j = 2i + 1) goes to slot j % 3, once the product
    // that read load j - 3 has completed: the last PV of item i - 2 (for K of item i) or the
    // last S of item i - 1 (for V of item i).
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int j = 0;
      bool ok = true;
      int4 nxt = first_item;
      for (int t = blockIdx.x; t < n_items && ok; t += grid) {
        const int4 it = nxt;
        if (t + grid < n_items) nxt = P.items[t + grid];
        const int g = it.x / P.nbk, b = it.x % P.nbk;
        for (int kv = 0; kv < 2; ++kv, ++j) {
          const int sl = j % KS;
          const uint32_t ph = static_cast<uint32_t>(j / KS) & 1;
          if (!mbar_wait(&kv_empty[sl], ph ^ 1, abort_flag, kKidKvOuter)) { ok = false; break; }
          uint64_t* full = kv ? &v_full[sl] : &k_full[sl];
          mbar_arrive_expect_tx(full, C::kKvBytes);
          for (int p = 0; p < C::kPanels; ++p)
            tma_load_3d(smem + C::kKvOff + sl * C::kKvBytes + p * C::kKvPanel, kv ? &tm_v : &tm_k, full, p * 64, g,
                        b * BK);
        }
      }
      // drain: the last load issued into each slot must land before the CTA exits (load L is
      // phase (L / 2) / 3 of its slot's K or V barrier)
      for (int x = 1; x <= KS; ++x) {
        const int L = j - x;
        if (L >= 0)
          mbar_wait((L & 1) ? &v_full[L % KS] : &k_full[L % KS], static_cast<uint32_t>((L >> 1) / KS) & 1, nullptr,
                    kKidKvOuter);
      }
    }
  } else if (warp == 2) {
    // ------------------------------ query gather ------------------------------
    // Lane q of the warp owns query q of the tile: it loads the CSR entry and issues that
    // query's boxes (RP / 8 boxes of 8 heads x all panels).
    if (lane == 0) tma_prefetch_desc(&tm_q);
    // every query row of the chunk is gathered once per block it chose, by CTAs working on
    // the same group at about the same time: keep the rows in L2 ahead of the streamed partials
    const uint64_t keep = l2_policy_evict_last();
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
            tma_load_4d_hint(dst + h8 * C::kGroupBytes, &tm_q, &q_full[qs], 0, g * P.R + h8 * 8, 0, e >> 5, keep);
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
  } else if (warp == 1 || warp == 3) {
    // ------------------------------ MMA issuers ------------------------------
    // warp 1: S(n) once its query rows and its item's K are in shared memory and PV(n - 3),
    //         which read P from the same TMEM columns, has completed.
    // warp 3: PV(n) once P(n) is written, its item's V is in shared memory and the epilogue
    //         has read O(n - 1) out of TMEM.
    if (lane == 0) {
      const bool is_s = (warp == 1);
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, BK, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, true);
      int n = 0, ni = 0;
      bool ok = true;
      int4 nxt = first_item;
      for (int t = blockIdx.x; t < n_items && ok; t += grid, ++ni) {
        const int4 it = nxt;
        if (t + grid < n_items) nxt = P.items[t + grid];
        const int ntiles = (it.z + TQ - 1) / TQ;
        const int sl = (2 * ni + (is_s ? 0 : 1)) % KS;            // slot of this item's K or V
        const uint32_t kv_addr = smem_u32(smem + C::kKvOff + sl * C::kKvBytes);
        // item ni's K (V) is the (ni / 3)-th K (V) block of its slot
        if (!mbar_wait(is_s ? &k_full[sl] : &v_full[sl], static_cast<uint32_t>(ni / KS) & 1, abort_flag, kKidKvOuter)) {
          ok = false;
          break;
        }
        for (int j = 0; j < ntiles; ++j, ++n) {
          const int w = n % NS;                                   // S/P region
          const uint32_t u = static_cast<uint32_t>(n / NS) & 1;   // phase parity of region w
          if (is_s) {
            const int qs = n % QS;
            if (!mbar_wait(&q_full[qs], static_cast<uint32_t>(n / QS) & 1, abort_flag, kKidKvOuter) ||
                !mbar_wait(&sp_free[w], u ^ 1, abort_flag, kKidKvOuter)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t q_addr = smem_u32(smem + C::kQOff + qs * C::kTileBytes);
            const uint32_t d_s = tmem + w * 128;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t adesc =
                  smem_desc(q_addr + (kk >> 2) * 1024 + (kk & 3) * 32, 16, C::kGroupBytes, kLayoutSw128);
              const uint64_t bdesc = smem_desc(kv_addr + (kk >> 2) * C::kKvPanel + (kk & 3) * 32, 16, 1024, kLayoutSw128);
              umma_bf16(d_s, adesc, bdesc, idesc_s, kk > 0);
            }
            umma_commit(&q_empty[qs]);
            umma_commit(&s_full[w]);
            if (j == ntiles - 1) umma_commit(&kv_empty[sl]);
          } else {
            if (!mbar_wait(&p_full[w], u, abort_flag, kKidKvOuter) ||
                !mbar_wait(o_free, (static_cast<uint32_t>(n) & 1) ^ 1, abort_flag, kKidKvOuter)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_o = tmem + kKvOCol;
            const uint32_t a_p = tmem + w * 128;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_bf16_ts(d_o, a_p + kk * 8, smem_desc(kv_addr + kk * 2048, C::kKvPanel, 1024, kLayoutSw128), idesc_o,
                           kk > 0);
            umma_commit(&sp_free[w]);
            umma_commit(o_full);
            if (j == ntiles - 1) umma_commit(&kv_empty[sl]);
          }
        }
      }
      // every product this thread issued completes before TMEM is released
      uint64_t* done = is_s ? s_done : pv_done;
      umma_commit(done);
      mbar_wait(done, 0, nullptr, kKidKvOuter);
    }
  } else if (warp >= kKvEpiWarp) {
    // ------------------------------ epilogue warpgroup ------------------------------
    // O of every tile: TMEM -> bf16 -> this warp's 32 rows of the swizzled staging tile; then
    // lane q of the warp issues the TMA stores of the warp's q-th query (2 KB: all its heads),
    // so each partial row leaves as whole lines. A warp reuses its staging rows once its own
    // stores have read them; the TMEM columns are handed back as soon as the last load lands.
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    constexpr int QPW = 32 / RP;                  // queries whose rows this warp holds
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t o_row = smem_u32(smem + C::kStgOff) + (m >> 3) * C::kGroupBytes + (m & 7) * 128;
    if (lane == 0) tma_prefetch_desc(&tm_o);
    // partials are read back only by the merge, after the whole chunk: evicted first
    const uint64_t stream_out = l2_policy_evict_first();
    int nt = 0;
    bool fail = false;
    int4 nxt = first_item;
    for (int t = blockIdx.x; t < n_items && !fail; t += grid) {
      const int4 it = nxt;
      if (t + grid < n_items) nxt = P.items[t + grid];
      const int g = it.x / P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        const int nq = min(TQ, it.z - j * TQ);
        const int qw = quad * QPW + lane;         // the query whose stores this lane issues
        const bool st_lane = (lane < QPW) && (qw < nq);
        const int e = st_lane ? __ldg(P.entries + it.y + j * TQ + qw) : 0;
        const uint32_t t_o = tmem + lane_base + kKvOCol;
        if (!mbar_wait(o_full, static_cast<uint32_t>(nt) & 1, abort_flag, kKidKvOuter)) { fail = true; break; }
        tc_fence_after();
        if (lane < QPW) bulk_wait_read_all();     // previous tile's stores have read the rows
        __syncwarp();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(t_o + c * 32, v);
          tmem_ld_wait();
          if (c == D / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
          }
#pragma unroll
          for (int x = 0; x < 4; ++x) {              // four 16-byte chunks of 8 columns
            const int ch = c * 4 + x;                // chunk index along d
            const uint32_t* s8 = v + x * 8;
            st_shared_v4(o_row + (ch >> 3) * 1024 + (((ch & 7) ^ (m & 7)) << 4),
                         pack_bf16x2(__uint_as_float(s8[0]), __uint_as_float(s8[1])),
                         pack_bf16x2(__uint_as_float(s8[2]), __uint_as_float(s8[3])),
                         pack_bf16x2(__uint_as_float(s8[4]), __uint_as_float(s8[5])),
                         pack_bf16x2(__uint_as_float(s8[6]), __uint_as_float(s8[7])));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (st_lane) {
          const int64_t il = static_cast<int64_t>(e >> 5) - P.row0;
          const int row = static_cast<int>((il * P.G + g) * P.k + (e & 31));
          const uint8_t* src = smem + C::kStgOff + qw * (RP / 8) * C::kGroupBytes;
          if (P.R >= 8) {
#pragma unroll
            for (int h8 = 0; h8 < RP / 8; ++h8)
              tma_store_4d_hint(&tm_o, src + h8 * C::kGroupBytes, 0, h8 * 8, 0, row, stream_out);
          } else {
#pragma unroll
            for (int p = 0; p < C::kPanels; ++p) tma_store_4d_hint(&tm_o, src + p * 1024, 0, 0, p, row, stream_out);
          }
          bulk_commit_group();
        }
      }
    }
    if (lane < QPW) bulk_wait_all();              // every store of this lane has completed
  } else if (warp >= 4) {
    // ------------------------------ softmax warpgroups ------------------------------
    // The four warps of a warpgroup never wait for one another: each hands its rows over
    // through mbarrier arrivals (P to the PV issuer).
    const int wg = (warp - 4) >> 2;               // takes tiles with nt % NW == wg
    const int quad = warp & 3;
    const int m = quad * 32 + lane;               // row of the tile == TMEM lane
    const int q = m / RP, r = m % RP;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
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
        if (nt % NW != wg) continue;
        const int sr = nt % NS;                     // S/P region of this tile
        const uint32_t u = static_cast<uint32_t>(nt / NS);
        const uint32_t t_s = t_lane + sr * 128;
        const int nq = min(TQ, it.z - j * TQ);
        const bool valid = (q < nq) && (r < P.R);
        const int e = (pref_nt == nt) ? e_pref : (valid ? __ldg(P.entries + it.y + j * TQ + q) : 0);
        const int i = valid ? (e >> 5) : 0;
        const int s = valid ? (e & 31) : 0;
        // load the entry for this warpgroup's next tile now (same item or the next one); rows
        // past that tile's queries read a neighbouring entry that is never used
        {
          int jn = j + NW;
          const int32_t* base = nullptr;
          if (jn < ntiles) {
            base = P.entries + it.y;
          } else if (t + grid < n_items && (jn -= ntiles) < (nxt.z + TQ - 1) / TQ) {
            base = P.entries + nxt.y;
          }
          pref_nt = base ? nt + NW : -1;
          if (base) e_pref = __ldg(base + jn * TQ + q);
        }
        const int limit = !valid ? -1 : ((b == i / BK) ? (i % BK) : BK - 1);   // keys c <= limit are visible
        // warps whose rows all see the whole block skip the per-key mask
        const bool whole = __all_sync(0xffffffffu, limit == BK - 1);
        // ---- row max (pass 1 over S; two 32-column loads per TMEM wait, 4 independent chains)
        if (!mbar_wait(&s_full[sr], u & 1, abort_flag, kKidKvOuter)) { fail = true; break; }
        tc_fence_after();
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        constexpr int LPW = (NCH >= 2) ? 2 : 1;   // 32-column loads per TMEM wait
#pragma unroll 1
        for (int c = 0; c < NCH; c += LPW) {
          uint32_t v[LPW][32];
#pragma unroll
          for (int h = 0; h < LPW; ++h) tmem_ld32(t_s + (c + h) * 32, v[h]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < LPW; ++h) {
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
        for (int c = 0; c < NCH; ++c) {
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
        if (lane == 0) mbar_arrive(&p_full[sr]);
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
