// Main Branch, KV-outer (KV-stationary) execution.
//
// hyper.ai "MiniMax Sparse Attention", Method (third paragraph): exact scaled dot-product
// softmax attention restricted to the tokens of the selected blocks; Key Contributions:
// KV-outer sparse attention keeps tensor cores busy under block-granular access and
// handles skewed block popularity without atomic updates (zhichai.net section 4.2).
//
// A work item is (group g, block b, up to kKvItemTiles tiles of the queries that chose b).
// A tile holds TQ = 128 / RP queries; query q of the tile occupies rows [q*RP, q*RP + R)
// of a 128-row operand (RP = max(R, 8) so every query starts on an 8-row swizzle atom).
// Per tile, with K_b / V_b resident in shared memory:
//   S = Q K_b^T            tcgen05.mma, M = 128 rows, N = 128 keys, K = d      -> TMEM
//   P = exp2(S*scale*log2e - rowmax)  (causal mask only when b is the query's own block)
//   O = P V_b              tcgen05.mma, M = 128, N = d, K = 128 keys            -> TMEM
//   partial (O / rowsum) -> bf16, and lse = rowmax + ln(rowsum), stored for the query's
//   slot s, so a later pass combines the k slots of every query (no atomics).
// Roles: warp 0 loads K_b/V_b (TMA), warp 2 gathers query rows (TMA, one box per query
// and 64-column panel), warp 1 issues the MMAs, warps 4..7 run softmax and the epilogue
// (one TMEM lane = one row per thread) and store partials with TMA.
#pragma once
#include "ptx.cuh"

namespace msa {

constexpr int kKvItemTiles = 8;
constexpr int kKvThreads = 256;

template <int D, int RP>
struct KvCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kPBytes = 128 * 128 * 2;
  static constexpr int TQ = 128 / RP;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kQOff = 2 * kTileBytes;   // 2 stages
  static constexpr int kPOff = 4 * kTileBytes;
  static constexpr int kOOff = kPOff + kPBytes;
  static constexpr int kBarOff = kOOff + kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;
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

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

template <int D, int RP>
__global__ void __launch_bounds__(kKvThreads, 1)
kvouter_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ KvParams P) {
  using C = KvCfg<D, RP>;
  constexpr int TQ = C::TQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* k_full = bars + 0;
  uint64_t* k_empty = bars + 1;
  uint64_t* v_full = bars + 2;
  uint64_t* v_empty = bars + 3;
  uint64_t* q_full = bars + 4;     // [2]
  uint64_t* q_empty = bars + 6;    // [2]
  uint64_t* s_full = bars + 8;     // [2]
  uint64_t* s_free = bars + 10;    // [2]
  uint64_t* o_full = bars + 12;    // [2]
  uint64_t* o_free = bars + 14;    // [2]
  uint64_t* p_full = bars + 16;
  uint64_t* p_empty = bars + 17;
  uint64_t* mma_done = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sm_fail = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1); mbar_init(k_empty, 1); mbar_init(v_full, 1); mbar_init(v_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 4);
      mbar_init(&o_full[i], 1); mbar_init(&o_free[i], 4);
    }
    mbar_init(p_full, 4); mbar_init(p_empty, 1); mbar_init(mma_done, 1);
    *abort_flag = 0;
    *sm_fail = 0;
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

  if (warp == 0) {
    // ------------------------------ K / V producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int ni = 0;
      for (int t = blockIdx.x; t < n_items; t += gridDim.x, ++ni) {
        const int4 it = P.items[t];
        const int g = it.x / P.nbk, b = it.x % P.nbk;
        if (!mbar_wait(k_empty, (ni & 1) ^ 1, abort_flag, kKidKvOuter)) break;
        mbar_arrive_expect_tx(k_full, C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(smem + C::kKOff + p * 16384, &tm_k, k_full, p * 64, g, b * 128);
        if (!mbar_wait(v_empty, (ni & 1) ^ 1, abort_flag, kKidKvOuter)) break;
        mbar_arrive_expect_tx(v_full, C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(smem + C::kVOff + p * 16384, &tm_v, v_full, p * 64, g, b * 128);
      }
      if (ni > 0) {  // drain the last loads
        mbar_wait(k_full, (ni - 1) & 1, nullptr, kKidKvOuter);
        mbar_wait(v_full, (ni - 1) & 1, nullptr, kKidKvOuter);
      }
    }
  } else if (warp == 2) {
    // ------------------------------ query gather ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int nt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_items && ok; t += gridDim.x) {
        const int4 it = P.items[t];
        const int g = it.x / P.nbk;
        const int ntiles = (it.z + TQ - 1) / TQ;
        for (int j = 0; j < ntiles; ++j, ++nt) {
          const int qs = nt & 1;
          if (!mbar_wait(&q_empty[qs], ((nt >> 1) & 1) ^ 1, abort_flag, kKidKvOuter)) { ok = false; break; }
          const int nq = min(TQ, it.z - j * TQ);
          mbar_arrive_expect_tx(&q_full[qs], nq * RP * 128 * C::kPanels);
          uint8_t* qs_base = smem + C::kQOff + qs * C::kTileBytes;
          for (int q = 0; q < nq; ++q) {
            const int e = __ldg(P.entries + it.y + j * TQ + q);
            const int i = e >> 5;
            for (int p = 0; p < C::kPanels; ++p)
              tma_load_3d(qs_base + p * 16384 + q * RP * 128, &tm_q, &q_full[qs], p * 64, g * P.R, i);
          }
        }
      }
      for (int b2 = 0; b2 < 2; ++b2) {
        if (nt > b2) {
          const int last = ((nt - 1 - b2) / 2) * 2 + b2;
          mbar_wait(&q_full[b2], (last >> 1) & 1, nullptr, kKidKvOuter);
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
      const uint32_t p_addr = smem_u32(smem + C::kPOff);
      int nt = 0, ni = 0;
      bool ok = true;
      // pending PV: tile counter, first / last tile of its item, item counter
      int pd_nt = -1, pd_first = 0, pd_last = 0, pd_ni = 0;
      auto issue_pv = [&](int tnt, int first, int last, int tni) -> bool {
        const int ob = tnt & 1;
        if (first && !mbar_wait(v_full, tni & 1, abort_flag, kKidKvOuter)) return false;
        if (!mbar_wait(p_full, tnt & 1, abort_flag, kKidKvOuter)) return false;
        if (!mbar_wait(&o_free[ob], ((tnt >> 1) & 1) ^ 1, abort_flag, kKidKvOuter)) return false;
        tc_fence_after();
        const uint32_t d_o = tmem + 256 + ob * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t adesc = smem_desc(p_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSw128);
          const uint64_t bdesc = smem_desc(v_addr + kk * 2048, 16384, 1024, kLayoutSw128);
          umma_bf16(d_o, adesc, bdesc, idesc_o, kk > 0);
        }
        umma_commit(p_empty);
        umma_commit(&o_full[ob]);
        if (last) umma_commit(v_empty);
        return true;
      };
      for (int t = blockIdx.x; t < n_items && ok; t += gridDim.x, ++ni) {
        const int4 it = P.items[t];
        const int ntiles = (it.z + TQ - 1) / TQ;
        if (!mbar_wait(k_full, ni & 1, abort_flag, kKidKvOuter)) { ok = false; break; }
        for (int j = 0; j < ntiles; ++j, ++nt) {
          const int qs = nt & 1, sb = nt & 1;
          if (!mbar_wait(&q_full[qs], (nt >> 1) & 1, abort_flag, kKidKvOuter)) { ok = false; break; }
          if (!mbar_wait(&s_free[sb], ((nt >> 1) & 1) ^ 1, abort_flag, kKidKvOuter)) { ok = false; break; }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(smem + C::kQOff + qs * C::kTileBytes);
          const uint32_t d_s = tmem + sb * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(d_s, smem_desc(q_addr + koff, 16, 1024, kLayoutSw128),
                      smem_desc(k_addr + koff, 16, 1024, kLayoutSw128), idesc_s, kk > 0);
          }
          umma_commit(&q_empty[qs]);
          umma_commit(&s_full[sb]);
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
    // ------------------------------ softmax + epilogue ------------------------------
    const int quad = warp & 3;
    const int m = quad * 32 + lane;          // row of the tile == TMEM lane
    const int q = m / RP, r = m % RP;
    const bool lead = (threadIdx.x == 128);
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* p_s = smem + C::kPOff;
    uint8_t* o_s = smem + C::kOOff;
    int nt = 0;
    bool fail = false;
    for (int t = blockIdx.x; t < n_items; t += gridDim.x) {
      const int4 it = P.items[t];
      const int g = it.x / P.nbk, b = it.x % P.nbk;
      const int ntiles = (it.z + TQ - 1) / TQ;
      bool stop = false;
      for (int j = 0; j < ntiles; ++j, ++nt) {
        const int nq = min(TQ, it.z - j * TQ);
        const bool valid = (q < nq) && (r < P.R);
        int i = 0, s = 0;
        if (valid) {
          const int e = __ldg(P.entries + it.y + j * TQ + q);
          i = e >> 5;
          s = e & 31;
        }
        const int sb = nt & 1;
        // ---- S -> registers
        if (!fail && !mbar_wait(&s_full[sb], (nt >> 1) & 1, abort_flag, kKidKvOuter)) fail = true;
        tc_fence_after();
        float x[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + sb * 128 + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) x[c * 32 + u] = __uint_as_float(v[u]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        // ---- softmax (exact within the block; the merge pass combines blocks)
        const int limit = !valid ? -1 : ((b == (i >> 7)) ? (i & 127) : 127);
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          x[c] = (c <= limit) ? x[c] * P.scale_log2 : -INFINITY;
          mx = fmaxf(mx, x[c]);
        }
        const float mref = (limit >= 0) ? mx : 0.0f;
        float l = 0.0f;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          x[c] = exp2f(x[c] - mref);   // masked -> 0
          l += x[c];
        }
        if (!fail && !mbar_wait(p_empty, (nt & 1) ^ 1, abort_flag, kKidKvOuter)) fail = true;
        {
          const uint32_t row_base = smem_u32(p_s) + m * 128;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint32_t addr = row_base + (c >> 3) * 16384 + (((c & 7) ^ (m & 7)) << 4);
            st_shared_v4(addr, pack_bf16x2(x[c * 8 + 0], x[c * 8 + 1]), pack_bf16x2(x[c * 8 + 2], x[c * 8 + 3]),
                         pack_bf16x2(x[c * 8 + 4], x[c * 8 + 5]), pack_bf16x2(x[c * 8 + 6], x[c * 8 + 7]));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // ---- O -> registers, normalise
        const int ob = nt & 1;
        if (!fail && !mbar_wait(&o_full[ob], (nt >> 1) & 1, abort_flag, kKidKvOuter)) fail = true;
        tc_fence_after();
        float o[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + 256 + ob * 128 + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) o[c * 32 + u] = __uint_as_float(v[u]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[ob]);
        const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
        // ---- staging (previous tile's stores must have read it)
        if (lead) bulk_wait_read_all();
        named_bar_sync(1, 128);
        {
          const uint32_t row_base = smem_u32(o_s) + m * 128;
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            const uint32_t addr = row_base + (c >> 3) * 16384 + (((c & 7) ^ (m & 7)) << 4);
            st_shared_v4(addr, pack_bf16x2(o[c * 8 + 0] * inv, o[c * 8 + 1] * inv),
                         pack_bf16x2(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv),
                         pack_bf16x2(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv),
                         pack_bf16x2(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv));
          }
        }
        if (valid) {
          const int64_t il = static_cast<int64_t>(i) - P.row0;
          P.lse[((il * P.G + g) * P.k + s) * P.R + r] = (mx + __log2f(l)) * 0.69314718055994531f;
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (lead) {
          for (int qq = 0; qq < nq; ++qq) {
            const int e = __ldg(P.entries + it.y + j * TQ + qq);
            const int64_t il = static_cast<int64_t>(e >> 5) - P.row0;
            const int row = static_cast<int>((il * P.G + g) * P.k + (e & 31));
            for (int p = 0; p < C::kPanels; ++p) tma_store_3d(&tm_o, o_s + p * 16384 + qq * RP * 128, p * 64, 0, row);
          }
          bulk_commit_group();
        }
        // ---- uniform stop decision across the four softmax warps
        if (fail && lane == 0) *sm_fail = 1;
        named_bar_sync(1, 128);
        if (*sm_fail) stop = true;
        named_bar_sync(1, 128);
        if (stop) break;
      }
      if (stop) break;
    }
    if (lead) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace msa
