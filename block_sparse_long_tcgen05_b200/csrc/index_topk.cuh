// Index Branch in one kernel: token scores, Block Max Pooling and the exp-free Top-k.
//
// hyper.ai "MiniMax Sparse Attention", Method (second paragraph): per GQA group, score every
// visible key token with the dot product of the index query and the shared index key, pool
// the scores to Bk = 128 blocks with a max, keep the Top-K blocks with the local block always
// included; zhichai.net section 4.1: selection needs only the order of the scores, so no exp
// is taken.
//
// TMA -> tcgen05.mma -> TMEM, persistent: a work item is one 128-query tile qa of one group
// over all the key tiles its rows need, two key tiles per step: one M = 128, N = 256 MMA chain
// (K = d_idx) per step into a double-buffered 256-column TMEM accumulator. (Issuing the same
// work as 128 x 128 MMAs measured ~20% slower: the issue of a tcgen05.mma takes about as
// long as a 128 x 128 x 16 product, so the wider instruction keeps the tensor pipe fed.)
// Eight epilogue warps: each TMEM lane quadrant is read by two warps, one per key tile of the
// step, and every thread keeps the best k - 1 blocks of its half of the row in registers
// (ordered score, block id); when the item ends the odd-tile half hands its list to the
// even-tile half through shared memory, which merges it and writes the row's block_ids. No
// token scores or block maxima reach memory.
// Items are ordered group-major (one group's index keys, N * d_idx * 2 bytes, are streamed
// by all CTAs at once), with the tiles of successive groups in alternating cost order, and
// dealt to CTAs in snake order (alternating direction every round) so the per-CTA sums of
// cost stay even.
//
// Block sizes BK in {32, 64, 128}: one 128-key tile holds F = 128 / BK blocks and the
// epilogue takes F segment maxima per tile. A query row needs every block before its own,
// and with F > 1 some of those lie in the key tile of the row's own query tile (the diagonal
// tile): the items then also score that tile, and each row keeps only the blocks
// b < floor(i / BK). Those blocks end before the row's own block, so no token mask is needed.
#pragma once
#include "index_blockmax.cuh"
#include "topk.cuh"

namespace msa {

struct IdxTopkParams {
  int nt;              // 128-query tiles of the sequence
  int G, k;
  int64_t N;
  int32_t* block_ids;  // [N, G, k]
};

// A work item is one 128-query tile qa of one group over all the key tiles it needs
// (kbend = qa + diag), taken two key tiles per step: one M = 128, N = 256 MMA chain per step,
// so each tcgen05.mma instruction carries twice the work of a 128 x 128 one.
struct IdxTopkItem {
  int g, qa, kbend;
};

// item t: group-major; within a group the tiles run in alternating directions (the last group
// descending), so the cost of consecutive items never jumps and the list ends with the
// cheapest items
// (diag = 1 when the diagonal key tile is scored, i.e. for block sizes below 128)
__device__ __forceinline__ IdxTopkItem idx_topk_item(const IdxTopkParams& P, int t, int diag) {
  IdxTopkItem it;
  it.g = t / P.nt;
  const int pr = t - it.g * P.nt;
  it.qa = ((P.G - 1 - it.g) & 1) ? pr : P.nt - 1 - pr;
  it.kbend = it.qa + diag;
  return it;
}

// CTA c's r-th item in snake order, or -1 when the round has none for it
__device__ __forceinline__ int idx_topk_slot(int r, int total) {
  const int grid = static_cast<int>(gridDim.x);
  const int t = r * grid + ((r & 1) ? grid - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x));
  return t < total ? t : -1;
}

// Insert (u, b) into a list sorted by (u descending, b ascending), whatever the order the
// candidates come in (the merge of the two halves of a row).
template <int KM>
__device__ __forceinline__ void topk_insert_any(uint32_t (&Ls)[KM], int (&Lb)[KM], uint32_t u, int b) {
  auto better = [](uint32_t ua, int ba, uint32_t ub, int bb) { return ua > ub || (ua == ub && ba < bb); };
  if (better(u, b, Ls[KM - 1], Lb[KM - 1])) {
#pragma unroll
    for (int p = KM - 1; p > 0; --p) {
      const bool down = better(u, b, Ls[p - 1], Lb[p - 1]);
      const bool here = better(u, b, Ls[p], Lb[p]);
      Ls[p] = down ? Ls[p - 1] : (here ? u : Ls[p]);
      Lb[p] = down ? Lb[p - 1] : (here ? b : Lb[p]);
    }
    if (better(u, b, Ls[0], Lb[0])) {
      Ls[0] = u;
      Lb[0] = b;
    }
  }
}

// Shared memory: one query tile, a ring of stages of two key tiles each ([panel][256 keys]
// [row bytes], so one descriptor covers both), the list exchange of the two row halves
// ([KM][128] scores and ids), barriers.
template <int DI, int KM>
struct IdxTopkCfg {
  using C = IdxCfg<DI>;
  static constexpr int kStages = (DI >= 128) ? 2 : 3;
  static constexpr int kKPanelBytes = 2 * C::kPanelBytes;
  static constexpr int kStageBytes = C::kPanels * kKPanelBytes;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = C::kTileBytes;
  static constexpr int kXOff = kKOff + kStages * kStageBytes;
  static constexpr int kBarOff = kXOff + KM * 128 * 8;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
};

template <int DI, int KM, int BK>
__global__ void __launch_bounds__(kIdxThreads, 1)
index_topk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ IdxTopkParams P) {
  using C = IdxCfg<DI>;
  using T = IdxTopkCfg<DI, KM>;
  constexpr int S = T::kStages;
  static_assert(T::kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(KM >= 1, "at least one non-local place");
  static_assert(BK == 32 || BK == 64 || BK == 128, "block size");
  constexpr int F = 128 / BK;               // blocks per 128-key tile
  constexpr int kDiag = (F > 1) ? 1 : 0;    // the diagonal key tile holds needed blocks
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;              // [S]
  uint64_t* k_empty = bars + 2 + S;         // [S]
  uint64_t* acc_full = bars + 2 + 2 * S;    // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* x_ready = acc_empty + 2;        // odd-tile half of each row's list written (4 warps)
  uint64_t* x_free = x_ready + 1;           // even-tile half has read it (4 warps)
  uint64_t* mma_done = x_free + 1;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  WaitCtl* abort_flag = reinterpret_cast<WaitCtl*>(tmem_base_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < S; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 8); }
    mbar_init(x_ready, 4);
    mbar_init(x_free, 4);
    mbar_init(mma_done, 1);
    wait_ctl_init(abort_flag);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int total = P.G * P.nt;
  const int rounds = (total + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      int64_t ik = 0;
      int n_item = 0;
      bool ok = true;
      for (int r = 0; r < rounds && ok; ++r) {
        const int t = idx_topk_slot(r, total);
        if (t < 0) continue;
        const IdxTopkItem it = idx_topk_item(P, t, kDiag);
        if (it.kbend == 0) continue;
        if (!mbar_wait(q_empty, (static_cast<uint32_t>(n_item) & 1) ^ 1, abort_flag, kKidIndexScore)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, C::kTileBytes);
        for (int pnl = 0; pnl < C::kPanels; ++pnl)
          tma_load_3d(smem + T::kQOff + pnl * C::kPanelBytes, &tm_q, q_full, pnl * C::kPanelElems, it.g, it.qa * 128);
        ++n_item;
        for (int kb = 0; kb < it.kbend; kb += 2, ++ik) {
          const int s = static_cast<int>(ik % S);
          const uint32_t u = static_cast<uint32_t>(ik / S);
          if (!mbar_wait(&k_empty[s], (u & 1) ^ 1, abort_flag, kKidIndexScore)) { ok = false; break; }
          const int ntile = (kb + 1 < it.kbend) ? 2 : 1;   // the second tile of the last step may not be needed
          uint8_t* ks = smem + T::kKOff + s * T::kStageBytes;
          mbar_arrive_expect_tx(&k_full[s], ntile * C::kTileBytes);
          for (int x = 0; x < ntile; ++x)
            for (int pnl = 0; pnl < C::kPanels; ++pnl)
              tma_load_3d(ks + pnl * T::kKPanelBytes + x * C::kPanelBytes, &tm_k, &k_full[s], pnl * C::kPanelElems, it.g,
                          (kb + x) * 128);
        }
      }
      // Drain: every TMA load this thread issued must land before the CTA exits.
      for (int s = 0; s < S; ++s) {
        if (ik > s) {
          const int64_t last = ((ik - 1 - s) / S) * S + s;
          mbar_wait(&k_full[s], static_cast<uint32_t>(last / S) & 1, nullptr, kKidIndexScore);
        }
      }
      if (n_item > 0) mbar_wait(q_full, static_cast<uint32_t>(n_item - 1) & 1, nullptr, kKidIndexScore);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false);
      int64_t ik = 0;
      int n_item = 0;
      bool ok = true;
      const uint32_t q_addr = smem_u32(smem + T::kQOff);
      for (int r = 0; r < rounds && ok; ++r) {
        const int t = idx_topk_slot(r, total);
        if (t < 0) continue;
        const IdxTopkItem it = idx_topk_item(P, t, kDiag);
        if (it.kbend == 0) continue;
        if (!mbar_wait(q_full, static_cast<uint32_t>(n_item) & 1, abort_flag, kKidIndexScore)) { ok = false; break; }
        ++n_item;
        tc_fence_after();
        for (int kb = 0; kb < it.kbend; kb += 2, ++ik) {
          const int s = static_cast<int>(ik % S);
          const uint32_t u = static_cast<uint32_t>(ik / S);
          const int ab = static_cast<int>(ik & 1);
          const uint32_t au = static_cast<uint32_t>(ik >> 1);
          if (!mbar_wait(&k_full[s], u & 1, abort_flag, kKidIndexScore)) { ok = false; break; }
          if (!mbar_wait(&acc_empty[ab], (au & 1) ^ 1, abort_flag, kKidIndexScore)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + T::kKOff + s * T::kStageBytes);
          const uint32_t d = tmem + ab * 256;
#pragma unroll
          for (int kk = 0; kk < C::kKSteps; ++kk) {
            const uint32_t kcol = (kk * 32) % C::kRowBytes;
            const uint32_t koff = (kk * 32) / C::kRowBytes * C::kPanelBytes + kcol;
            const uint32_t kofb = (kk * 32) / C::kRowBytes * T::kKPanelBytes + kcol;
            umma_bf16(d, smem_desc(q_addr + koff, 16, C::kSbo, C::kLayout), smem_desc(k_addr + kofb, 16, C::kSbo, C::kLayout),
                      idesc, kk > 0);
          }
          umma_commit(&k_empty[s]);
          umma_commit(&acc_full[ab]);
        }
        umma_commit(q_empty);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, kKidIndexScore);
    }
  } else {
    // ------------------------------ epilogue: block max + running Top-k ------------------------------
    // Eight warps: the four TMEM lane quadrants, each read by two warps, one per key tile of
    // the step (half 0: even key tiles, columns 0-127; half 1: odd ones, columns 128-255).
    // Each thread keeps the best k - 1 blocks of its half of the row; at the end of the item
    // half 1 hands its list over through shared memory and half 0 merges and writes the row.
    const int ew = warp - 2;                 // 0..7
    const int half = ew >> 2;
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    uint32_t* xs = reinterpret_cast<uint32_t*>(smem + T::kXOff);   // [KM][128] scores
    int* xb = reinterpret_cast<int*>(xs + KM * 128);                // [KM][128] block ids
    int64_t ik = 0;
    int n_end = 0;   // items ended (list exchanges)
    bool ok = true;
    for (int r = 0; r < rounds && ok; ++r) {
      const int t = idx_topk_slot(r, total);
      if (t < 0) continue;
      const IdxTopkItem it = idx_topk_item(P, t, kDiag);
      const int qb = it.qa;
      const int64_t i = static_cast<int64_t>(qb) * 128 + row;
      const int bl = static_cast<int>(i / BK);   // this row's local block
      // running top list: ordered scores (descending) and their block ids; 0 is below every
      // real ordered score
      uint32_t Ls[KM];
      int Lb[KM];
#pragma unroll
      for (int p = 0; p < KM; ++p) { Ls[p] = 0u; Lb[p] = -1; }
      // Blocks that beat the list's current last entry wait in a CB-entry buffer (ascending
      // block order) and go into the list together when some row of the warp has CB: the
      // insertion network, which the whole warp runs whenever any row needs it, then runs
      // about as often as the busiest row has candidates instead of whenever any row has one
      // (measured: 8 and 16 entries are slower than 4).
      constexpr int CB = 4;
      uint32_t cu[CB];
      int cb[CB];
      int nc = 0;
      auto flush = [&]() {
#pragma unroll
        for (int c = 0; c < CB; ++c)
          if (c < nc) topk_insert_ascending<KM>(Ls, Lb, cu[c], cb[c]);
        nc = 0;
      };
      // offer block b with segment maximum m (blocks arrive in ascending order)
      auto offer = [&](float m, int b, bool valid) {
        m = __fadd_rn(m, 0.0f);   // -0 -> +0 so equal scores give equal keys
        uint32_t u = __float_as_uint(m);
        u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        if (valid && u > Ls[KM - 1]) {
#pragma unroll
          for (int c = 0; c < CB; ++c)
            if (nc == c) { cu[c] = u; cb[c] = b; }
          ++nc;
        }
        if (__any_sync(0xffffffffu, nc == CB)) flush();
      };
      for (int kb0 = 0; kb0 < it.kbend; kb0 += 2, ++ik) {
        const int kb = kb0 + half;               // this warp's key tile of the step
        const int ab = static_cast<int>(ik & 1);
        const uint32_t au = static_cast<uint32_t>(ik >> 1);
        if (!mbar_wait(&acc_full[ab], au & 1, abort_flag, kKidIndexScore)) { ok = false; break; }
        tc_fence_after();
        if (kb < qb + kDiag) {
          const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + ab * 256 + half * 128;
          // the 128-column row in two halves: the first half's max chains run while the second
          // half is in flight, then the accumulator is handed back
          uint32_t v[4][32];
          tmem_ld32(taddr, v[0]);
          tmem_ld32(taddr + 32, v[1]);
          tmem_ld_wait();
          tmem_ld32(taddr + 64, v[2]);
          tmem_ld32(taddr + 96, v[3]);
          if constexpr (F == 1) {
            float m8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) m8[j] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int j = 0; j < 32; j += 2)
                m8[(c * 16 + (j >> 1)) & 7] =
                    max3f(m8[(c * 16 + (j >> 1)) & 7], __uint_as_float(v[c][j]), __uint_as_float(v[c][j + 1]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
#pragma unroll
            for (int c = 2; c < 4; ++c)
#pragma unroll
              for (int j = 0; j < 32; j += 2)
                m8[(c * 16 + (j >> 1)) & 7] =
                    max3f(m8[(c * 16 + (j >> 1)) & 7], __uint_as_float(v[c][j]), __uint_as_float(v[c][j + 1]));
            offer(fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))),
                  kb, true);
          } else {
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
            constexpr int CPS = BK / 32;     // 32-column chunks per block
#pragma unroll
            for (int f = 0; f < F; ++f) {
              float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
              for (int c = f * CPS; c < (f + 1) * CPS; ++c)
#pragma unroll
                for (int j = 0; j < 32; j += 2)
                  m4[(j >> 1) & 3] = max3f(m4[(j >> 1) & 3], __uint_as_float(v[c][j]), __uint_as_float(v[c][j + 1]));
              const int b = kb * F + f;
              offer(fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])), b, b < bl);
            }
          }
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
      }
      if (!ok) continue;
      flush();
      // ---- the two halves of each row: half 1 writes its list, half 0 merges it
      const uint32_t xp = static_cast<uint32_t>(n_end) & 1;
      ++n_end;
      if (half == 1) {
        if (!mbar_wait(x_free, xp ^ 1, abort_flag, kKidIndexScore)) { ok = false; continue; }
#pragma unroll
        for (int p = 0; p < KM; ++p) { xs[p * 128 + row] = Ls[p]; xb[p * 128 + row] = Lb[p]; }
        __syncwarp();
        if (lane == 0) mbar_arrive(x_ready);
        continue;
      }
      if (!mbar_wait(x_ready, xp, abort_flag, kKidIndexScore)) { ok = false; continue; }
#pragma unroll
      for (int p = 0; p < KM; ++p) topk_insert_any<KM>(Ls, Lb, xs[p * 128 + row], xb[p * 128 + row]);
      __syncwarp();
      if (lane == 0) mbar_arrive(x_free);
      if (i >= P.N) continue;
      int32_t* out = P.block_ids + (i * P.G + it.g) * P.k;
      if (bl + 1 <= P.k) {
        topk_all_visible(bl, P.k, out);
      } else {
        int ids[KM];
#pragma unroll
        for (int p = 0; p < KM; ++p) ids[p] = Lb[p];
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace msa
