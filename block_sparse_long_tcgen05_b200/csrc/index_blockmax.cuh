// Index Branch, part 1: token scores with the block max fused into the epilogue.
//
// hyper.ai "MiniMax Sparse Attention", Method (second paragraph): each GQA group scores
// every visible key token with a dot product of its index query and the shared index key,
// and Block Max Pooling reduces the token scores of each Bk = 128 block to one value.
//
// One launch covers the query blocks [qb0, qb1) of one sequence, all groups. For query
// block qb only the blocks kb < qb are scored: the query's own (local) block is always
// selected, so its score is never needed, and every block before it lies entirely in
// the causal past of all 128 queries of qb, so no mask is needed either.
//
// Execution (one persistent CTA per SM):
//   * work item = (group g, query-block pair {qa, qa+1}, run of up to kKbRun key blocks);
//     items are ordered group-major, then by key run, then by pair, and dealt to CTAs
//     round-robin, so at any moment the CTAs stream the same few key tiles (L2 reuse)
//     while each keeps its own two query tiles resident;
//   * warp 0 issues TMA loads (query tiles double-buffered, key tiles in a kStages ring);
//   * warp 1 issues tcgen05.mma (M = 128 queries, N = 128 keys, K = d_idx, bf16 -> fp32)
//     for both query tiles against each key tile, into double-buffered TMEM accumulators;
//   * warps 2..9 drain TMEM (one row per thread), take the row max over the 128 keys,
//     and write it as an order-preserving uint32 key.
//
// Output layout (per group g, for the launch's query blocks): block qb owns a region of
// qb * 128 uint32 entries, entry (kb, r) at kb * 128 + r, r = row within the query
// block; regions follow each other in qb order. Each warp therefore writes 128
// contiguous bytes per key block.
#pragma once
#include "ptx.cuh"

namespace msa {

constexpr int kIdxKbRun = 64;     // key blocks per work item
constexpr int kIdxStages = 3;     // key-tile ring depth
constexpr int kIdxMaxRuns = 512;  // max key runs per launch (qb1 <= 512 * 64 = 32768 blocks)
constexpr int kIdxThreads = 320;  // 10 warps

struct IdxRunTable {
  // For key run c (key blocks [c * kIdxKbRun, ...)): the first pair that reaches it and
  // the number of items of all runs before it (per group).
  int pmin[kIdxMaxRuns];
  int prefix[kIdxMaxRuns + 1];
};

struct IdxParams {
  int qb0, qb1;            // query blocks of this launch
  int npairs;              // ceil((qb1 - qb0) / 2)
  int nruns;               // key runs
  int G;
  int64_t items_per_group;
  int64_t region_per_group;  // uint32 entries per group in `maxima`
  uint32_t* maxima;
};

template <int DI>
struct IdxCfg {
  static constexpr bool kSw64 = (DI == 32);
  static constexpr int kRowBytes = kSw64 ? 64 : 128;          // bytes per row per panel
  static constexpr int kPanels = kSw64 ? 1 : DI / 64;
  static constexpr int kPanelBytes = 128 * kRowBytes;         // 128 rows
  static constexpr int kTileBytes = kPanels * kPanelBytes;    // = 128 * DI * 2
  static constexpr int kPanelElems = kRowBytes / 2;           // elements per panel row
  static constexpr uint32_t kLayout = kSw64 ? kLayoutSw64 : kLayoutSw128;
  static constexpr uint32_t kSbo = 8 * kRowBytes;             // 8-row group stride
  static constexpr int kKSteps = DI / 16;
  // smem: Q [2 bufs][2 tiles], K [stages], then barriers
  static constexpr int kQOff = 0;
  static constexpr int kKOff = 4 * kTileBytes;
  static constexpr int kBarOff = kKOff + kIdxStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;     // + alignment slack
};

struct IdxItem {
  int g, qa, has_b, kb_begin, kb_end;
};

__device__ __forceinline__ IdxItem idx_decode_item(const IdxParams& P, const IdxRunTable& T, int64_t t) {
  IdxItem it;
  it.g = static_cast<int>(t / P.items_per_group);
  int rem = static_cast<int>(t - static_cast<int64_t>(it.g) * P.items_per_group);
  // find run c with prefix[c] <= rem < prefix[c+1] (binary search)
  int lo = 0, hi = P.nruns - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (T.prefix[mid] <= rem) lo = mid; else hi = mid - 1;
  }
  const int c = lo;
  const int p = T.pmin[c] + (rem - T.prefix[c]);
  it.qa = P.qb0 + 2 * p;
  it.has_b = (it.qa + 1 < P.qb1) ? 1 : 0;
  const int kbend = it.has_b ? it.qa + 1 : it.qa;
  it.kb_begin = c * kIdxKbRun;
  it.kb_end = min(kbend, it.kb_begin + kIdxKbRun);
  return it;
}

// Region start (uint32 entries) of query block qb inside its group's part of `maxima`.
__device__ __forceinline__ int64_t idx_region(int qb, int qb0) {
  return 128ll * ((static_cast<int64_t>(qb) * (qb - 1)) / 2 - (static_cast<int64_t>(qb0) * (qb0 - 1)) / 2);
}

template <int DI>
__global__ void __launch_bounds__(kIdxThreads, 1)
index_blockmax_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ IdxParams P, const __grid_constant__ IdxRunTable T) {
  using C = IdxCfg<DI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars + 0;              // [2]
  uint64_t* q_empty = bars + 2;             // [2]
  uint64_t* k_full = bars + 4;              // [stages]
  uint64_t* k_empty = bars + 4 + kIdxStages;
  uint64_t* acc_full = bars + 4 + 2 * kIdxStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;               // [2]
  uint64_t* mma_done = acc_empty + 2;               // [1]
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  WaitCtl* abort_flag = reinterpret_cast<WaitCtl*>(tmem_base_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1); }
    for (int i = 0; i < kIdxStages; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 8); }
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

  const int64_t total = P.items_per_group * P.G;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      int64_t ik = 0;
      int n_item = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x, ++n_item) {
        const IdxItem it = idx_decode_item(P, T, t);
        const int qbuf = n_item & 1;
        const uint32_t qu = static_cast<uint32_t>(n_item >> 1);
        if (!mbar_wait(&q_empty[qbuf], (qu & 1) ^ 1, abort_flag, kKidIndexScore)) { ok = false; break; }
        uint8_t* qa_s = smem + C::kQOff + (qbuf * 2 + 0) * C::kTileBytes;
        uint8_t* qb_s = smem + C::kQOff + (qbuf * 2 + 1) * C::kTileBytes;
        mbar_arrive_expect_tx(&q_full[qbuf], (it.has_b ? 2 : 1) * C::kTileBytes);
        for (int pnl = 0; pnl < C::kPanels; ++pnl) {
          tma_load_3d(qa_s + pnl * C::kPanelBytes, &tm_q, &q_full[qbuf], pnl * C::kPanelElems, it.g, it.qa * 128);
          if (it.has_b)
            tma_load_3d(qb_s + pnl * C::kPanelBytes, &tm_q, &q_full[qbuf], pnl * C::kPanelElems, it.g,
                        (it.qa + 1) * 128);
        }
        for (int kb = it.kb_begin; kb < it.kb_end; ++kb, ++ik) {
          const int s = static_cast<int>(ik % kIdxStages);
          const uint32_t u = static_cast<uint32_t>(ik / kIdxStages);
          if (!mbar_wait(&k_empty[s], (u & 1) ^ 1, abort_flag, kKidIndexScore)) { ok = false; break; }
          uint8_t* ks = smem + C::kKOff + s * C::kTileBytes;
          mbar_arrive_expect_tx(&k_full[s], C::kTileBytes);
          for (int pnl = 0; pnl < C::kPanels; ++pnl)
            tma_load_3d(ks + pnl * C::kPanelBytes, &tm_k, &k_full[s], pnl * C::kPanelElems, it.g, kb * 128);
        }
      }
      // Drain: every TMA load this thread issued must land before the CTA exits.
      for (int s = 0; s < kIdxStages; ++s) {
        if (ik > s) {
          const int64_t last = ((ik - 1 - s) / kIdxStages) * kIdxStages + s;
          mbar_wait(&k_full[s], static_cast<uint32_t>(last / kIdxStages) & 1, nullptr, kKidIndexScore);
        }
      }
      for (int b = 0; b < 2; ++b) {
        if (n_item > b) {
          const int last = ((n_item - 1 - b) / 2) * 2 + b;
          mbar_wait(&q_full[b], static_cast<uint32_t>(last >> 1) & 1, nullptr, kKidIndexScore);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      int64_t ik = 0;
      int n_item = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x, ++n_item) {
        const IdxItem it = idx_decode_item(P, T, t);
        const int qbuf = n_item & 1;
        const uint32_t qu = static_cast<uint32_t>(n_item >> 1);
        if (!mbar_wait(&q_full[qbuf], qu & 1, abort_flag, kKidIndexScore)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qa_addr = smem_u32(smem + C::kQOff + (qbuf * 2 + 0) * C::kTileBytes);
        const uint32_t qb_addr = smem_u32(smem + C::kQOff + (qbuf * 2 + 1) * C::kTileBytes);
        for (int kb = it.kb_begin; kb < it.kb_end; ++kb, ++ik) {
          const int s = static_cast<int>(ik % kIdxStages);
          const uint32_t u = static_cast<uint32_t>(ik / kIdxStages);
          const int ab = static_cast<int>(ik & 1);
          const uint32_t au = static_cast<uint32_t>(ik >> 1);
          if (!mbar_wait(&k_full[s], u & 1, abort_flag, kKidIndexScore)) { ok = false; break; }
          if (!mbar_wait(&acc_empty[ab], (au & 1) ^ 1, abort_flag, kKidIndexScore)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + C::kKOff + s * C::kTileBytes);
          const uint32_t d_a = tmem + ab * 256;
          const uint32_t d_b = d_a + 128;
          const bool a_active = kb < it.qa;
#pragma unroll
          for (int kk = 0; kk < C::kKSteps; ++kk) {
            const uint32_t koff = (kk * 32) / C::kRowBytes * C::kPanelBytes + (kk * 32) % C::kRowBytes;
            const uint64_t bdesc = smem_desc(k_addr + koff, 16, C::kSbo, C::kLayout);
            if (a_active) umma_bf16(d_a, smem_desc(qa_addr + koff, 16, C::kSbo, C::kLayout), bdesc, idesc, kk > 0);
            if (it.has_b) umma_bf16(d_b, smem_desc(qb_addr + koff, 16, C::kSbo, C::kLayout), bdesc, idesc, kk > 0);
          }
          umma_commit(&k_empty[s]);
          umma_commit(&acc_full[ab]);
        }
        umma_commit(&q_empty[qbuf]);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, kKidIndexScore);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int ew = warp - 2;                 // 0..7
    const int tile = ew >> 2;                // 0 = A (qa), 1 = B (qa + 1)
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    int64_t ik = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const IdxItem it = idx_decode_item(P, T, t);
      const int qb = it.qa + tile;
      const bool tile_present = (tile == 0) || it.has_b;
      uint32_t* out = P.maxima + static_cast<int64_t>(it.g) * P.region_per_group + idx_region(qb, P.qb0) + row;
      for (int kb = it.kb_begin; kb < it.kb_end; ++kb, ++ik) {
        const int ab = static_cast<int>(ik & 1);
        const uint32_t au = static_cast<uint32_t>(ik >> 1);
        if (!mbar_wait(&acc_full[ab], au & 1, abort_flag, kKidIndexScore)) { ok = false; break; }
        tc_fence_after();
        if (tile_present && kb < qb) {
          const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + ab * 256 + tile * 128;
          float m = -INFINITY;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(taddr + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j += 2) m = max3f(m, __uint_as_float(r[j]), __uint_as_float(r[j + 1]));
          }
          m = __fadd_rn(m, 0.0f);   // -0 -> +0 so equal scores give equal keys
          uint32_t u = __float_as_uint(m);
          u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
          out[static_cast<int64_t>(kb) * 128] = u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
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
