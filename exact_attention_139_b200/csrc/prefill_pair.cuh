// prefill_pair.cuh -- forward (prefill) attention with each tensor-core product spanning a pair of
// SMs (tcgen05 cta_group::2), for d = dv = 128, dense key ranges, even GQA groups.
//
// Arithmetic as in prefill2.cuh (the standard flow S = Q.K^T, P = softmax(S), O = P.V of the
// FlashMLA-ETAP summary, "Mecanismo Central", item 1, tile by tile on chip). What changes is the
// split of the work over the hardware:
//   * a cluster of two CTAs takes a work unit of two 256-row query tiles: rows [q0, q0 + 256) of
//     sibling query heads h (tile A) and h + 1 (tile B) of one kv head; the even CTA owns rows
//     q0.., the odd CTA rows q0 + 128..;
//   * every product is one M = 256 tcgen05.mma issued by the even CTA: A rows come from each CTA's
//     own Q (S) or P in TMEM (P.V), the B operand is split by halves of N (for S each CTA holds 64
//     of the 128 keys of a key tile, for P.V 64 of the 128 dv columns of V), and each CTA's TMEM
//     receives its 128 rows of S and O. One issued instruction carries twice the math of the
//     single-SM kernel, whose single issuing thread could not keep up with M = 128 products;
//   * each CTA runs its own TMA producer and two softmax warpgroups exactly as in the single-SM
//     kernel (one query row per thread, P written back over S in TMEM); load completions are
//     counted on the even CTA's barriers, product completions are signalled to both CTAs'
//     barriers, and the odd CTA's softmax threads arrive on the even CTA's P-ready and O-free
//     barriers through shared::cluster addresses;
//   * under a causal mask the even CTA's rows see one key tile fewer than the odd CTA's on the
//     diagonal; the pair computes that tile for both (the even half is fully masked: p = 0).
// Warps: 0-7 softmax, 8 TMA producer, 9 TMEM allocator (+ MMA issuer in the even CTA).
#pragma once

#include "prefill2.cuh"

namespace attn {

struct PairCfg {
  static constexpr int D = 128, BN = 128;
  static constexpr int CHUNK = 128 * 128;            // 128 rows x 64 columns of 16-bit, swizzled
  static constexpr int Q_BYTES = 2 * CHUNK;          // this CTA's 128 rows x 128 d of one tile
  static constexpr int KCHUNK = 64 * 128;            // 64 keys x 64 columns
  static constexpr int KH_BYTES = 2 * KCHUNK;        // this CTA's 64 keys x 128 d of K_j
  static constexpr int VH_BYTES = CHUNK;             // 128 keys x this CTA's 64 dv columns of V_j
  static constexpr int STAGE_BYTES = KH_BYTES + VH_BYTES;
  static constexpr int NS = 4;
  static constexpr int OFF_Q = 0;                    // Q_A, then Q_B
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * STAGE_BYTES;
  // q_full, q_empty, kv_full[NS], kv_empty[NS], s_full[2], p_full[2], o_ready[2], o_free[2], drain
  static constexpr int N_BARS = 2 + 2 * NS + 8 + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  __host__ __device__ static constexpr uint32_t s_col(int x) { return (uint32_t)(128 * x); }
  __host__ __device__ static constexpr uint32_t o_col(int x) { return (uint32_t)(256 + 128 * x); }
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Unit u of the pair kernel: (batch, head pair, 256-row level), levels heaviest first inside
// groups of group_b batches (the order of prefill_unit with 256-row levels and head pairs).
__device__ __forceinline__ UnitCoords pair_unit(const Prefill2Params& p, int u) {
  const int n_lvl = p.n_pairs;  // ceil(ceil(Lq / 128) / 2) levels of 256 rows
  const int hpl = p.Hq / 2;
  const int per_group = p.group_b * n_lvl * hpl;
  const int g = u / per_group;
  const int b0 = g * p.group_b;
  const int gb = min(p.group_b, p.B - b0);
  const int w = u - g * per_group;
  const int lvl = w / (gb * hpl);
  const int rem = w - lvl * gb * hpl;
  UnitCoords c;
  c.b = b0 + rem / hpl;
  c.h = 2 * (rem % hpl);
  c.q0 = (n_lvl - 1 - lvl) * 256;
  return c;
}

template <typename E>
__global__ void __launch_bounds__(PairCfg::THREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kh,
                        const __grid_constant__ CUtensorMap tm_v, const Prefill2Params p) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: even CTA (issues the products), 1: odd CTA
  const int pair = blockIdx.x >> 1, n_pairs_grid = gridDim.x >> 1;

  const uint32_t bar_q_full = base + C::OFF_BAR;
  const uint32_t bar_q_empty = bar_q_full + 8;
  const uint32_t bar_kv_full = bar_q_empty + 8;
  const uint32_t bar_kv_empty = bar_kv_full + 8 * C::NS;
  const uint32_t bar_s_full = bar_kv_empty + 8 * C::NS;  // [2]
  const uint32_t bar_p_full = bar_s_full + 16;           // [2]
  const uint32_t bar_o_ready = bar_p_full + 16;          // [2]
  const uint32_t bar_o_free = bar_o_ready + 16;          // [2]
  const uint32_t bar_drain = bar_o_free + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_kv_full + 8 * s, 1);
      mbar_init(bar_kv_empty + 8 * s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_s_full + 8 * x, 1);
      mbar_init(bar_p_full + 8 * x, 256);  // both CTAs' 128 softmax threads
      mbar_init(bar_o_ready + 8 * x, 1);
      mbar_init(bar_o_free + 8 * x, 256);
    }
    mbar_init(bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  __syncthreads();
  cluster_sync_all();  // the other CTA's barriers are initialised before anything reaches them
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 8) {
    // ------------------------------- TMA producer (both CTAs) -------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kh);
      tma_prefetch_desc(&tm_v);
      bool ok = true;
      int kv_t = 0, qc = 0;
      // both CTAs' load completions are counted on the even CTA's barriers
      const uint32_t q_full_lead = mapa_shared(bar_q_full, 0);
      for (int k = 0, u = pair; u < p.n_units && ok; ++k, u = prefill_unit_index(k, pair, n_pairs_grid)) {
        const UnitCoords uc = pair_unit(p, u);
        const int n = max(prefill_kv_tiles(p, uc.q0), prefill_kv_tiles(p, uc.q0 + 128));
        const int zkv = uc.b * p.Hkv + uc.h / p.G;
        if (qc > 0) ok = mbar_wait(bar_q_empty, (qc - 1) & 1, 62);
        if (!ok) break;
        // both tiles of both CTAs land on the even CTA's barrier
        if (rank == 0) mbar_arrive_expect_tx(bar_q_full, 4 * C::Q_BYTES);
        for (int x = 0; x < 2; ++x) {
          const int zq = uc.b * p.Hq + uc.h + x;
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(base + C::OFF_Q + x * C::Q_BYTES + c * C::CHUNK, &tm_q, q_full_lead,
                             64 * c, uc.q0 + 128 * (int)rank, zq);
        }
        ++qc;
        for (int j = 0; j < n && ok; ++j) {
          const int s = kv_t % C::NS;
          if (kv_t >= C::NS) ok = mbar_wait(bar_kv_empty + 8 * s, ((kv_t / C::NS) & 1) ^ 1, 61);
          if (!ok) break;
          const uint32_t full = bar_kv_full + 8 * s;
          const uint32_t full_lead = mapa_shared(full, 0);
          const uint32_t dst = base + C::OFF_KV + s * C::STAGE_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(full, 2 * C::STAGE_BYTES);
          // this CTA's half of K_j: keys j*128 + 64*rank .. +64, all 128 columns
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(dst + c * C::KCHUNK, &tm_kh, full_lead, 64 * c, j * C::BN + 64 * (int)rank,
                             zkv);
          // this CTA's half of V_j: all 128 keys, dv columns 64*rank .. +64
          tma_load_3d_pair(dst + C::KH_BYTES, &tm_v, full_lead, 64 * (int)rank, j * C::BN, zkv);
          ++kv_t;
        }
      }
      if (!ok && rank == 0) {
        // the even CTA's barriers count both CTAs' bytes: wait for what is in flight
        if (qc > 0) mbar_wait_drain(bar_q_full, (qc - 1) & 1);
        for (int u = max(0, kv_t - C::NS); u < kv_t; ++u) mbar_wait_drain(bar_kv_full + 8 * (u % C::NS), (u / C::NS) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------- MMA issuer (even CTA) -------------------------------
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_s = make_idesc(256, C::BN, false, false, E::kFmt);
      constexpr uint32_t idesc_o = make_idesc(256, C::D, false, true, E::kFmt);
      constexpr uint16_t kBoth = 0x3;
      bool ok = true, issued = false;
      int kv_t = 0, qc = 0;
      int p_cnt[2] = {0, 0}, units_done[2] = {0, 0};
      auto wait_stage = [&](int idx, uint32_t site) {
        ok = mbar_wait(bar_kv_full + 8 * (idx % C::NS), (idx / C::NS) & 1, site);
        if (ok) tc_fence_after();
      };
      auto issue_s = [&](int x, int sidx) {
        const uint32_t kb = base + C::OFF_KV + (sidx % C::NS) * C::STAGE_BYTES;
        const uint32_t qb = base + C::OFF_Q + x * C::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::D / 16; ++kk) {
          const uint64_t ad = make_sdesc(qb + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = make_sdesc(kb + (kk >> 2) * C::KCHUNK + (kk & 3) * 32, 16, 1024, kSwizzle128B);
          mma_ss_pair(tmem + C::s_col(x), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit_pair(bar_s_full + 8 * x, kBoth);
        issued = true;
      };
      for (int k = 0, u = pair; u < p.n_units && ok; ++k, u = prefill_unit_index(k, pair, n_pairs_grid)) {
        const UnitCoords uc = pair_unit(p, u);
        const int n = max(prefill_kv_tiles(p, uc.q0), prefill_kv_tiles(p, uc.q0 + 128));
        ok = mbar_wait(bar_q_full, qc & 1, 63);
        if (!ok) break;
        ++qc;
        tc_fence_after();
        wait_stage(kv_t, 64);
        if (!ok) break;
        issue_s(0, kv_t);
        issue_s(1, kv_t);
        if (n == 1) mma_commit_pair(bar_q_empty, kBoth);
        for (int j = 0; j < n && ok; ++j) {
          const int si = kv_t + j;
          bool next_ready = false;
          for (int x = 0; x < 2 && ok; ++x) {
            if (j == 0 && units_done[x] > 0) {
              ok = mbar_wait_cluster(bar_o_free + 8 * x, (units_done[x] - 1) & 1, 66);
              if (!ok) break;
            }
            ok = mbar_wait_cluster(bar_p_full + 8 * x, p_cnt[x] & 1, 67);
            if (!ok) break;
            ++p_cnt[x];
            tc_fence_after();
            const uint32_t vb = base + C::OFF_KV + (si % C::NS) * C::STAGE_BYTES + C::KH_BYTES;
#pragma unroll
            for (int kk = 0; kk < C::BN / 16; ++kk) {
              const uint64_t bd = make_sdesc(vb + kk * 2048, C::CHUNK, 1024, kSwizzle128B);
              mma_ts_pair(tmem + C::o_col(x), tmem + C::s_col(x) + 8 * kk, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            }
            if (x == 1) mma_commit_pair(bar_kv_empty + 8 * (si % C::NS), kBoth);
            if (j + 1 < n) {
              if (!next_ready) {
                wait_stage(si + 1, 68);
                if (!ok) break;
                next_ready = true;
              }
              issue_s(x, si + 1);
            } else {
              mma_commit_pair(bar_o_ready + 8 * x, kBoth);
              ++units_done[x];
            }
          }
          if (!ok) break;
          if (j == n - 2) mma_commit_pair(bar_q_empty, kBoth);
        }
        if (!ok) break;
        kv_t += n;
      }
      if (!ok && issued) {
        mma_commit_pair(bar_drain, 0x1);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // --------------------------- softmax warpgroups (both CTAs) ---------------------------
    const int x = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t tw = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = C::s_col(x), o_col = C::o_col(x);
    // where this thread's P-ready and O-free arrivals go: the even CTA's barriers
    const uint32_t p_full_l = bar_p_full + 8 * x, o_free_l = bar_o_free + 8 * x;
    const uint32_t p_full_c = mapa_shared(p_full_l, 0), o_free_c = mapa_shared(o_free_l, 0);
    const float c2 = p.scale_log2;
    const int off = p.Lk - p.Lq;
    int s_cnt = 0, o_cnt = 0;
    bool ok = true;
    for (int k = 0, u = pair; u < p.n_units && ok; ++k, u = prefill_unit_index(k, pair, n_pairs_grid)) {
      const UnitCoords uc = pair_unit(p, u);
      const int n = max(prefill_kv_tiles(p, uc.q0), prefill_kv_tiles(p, uc.q0 + 128));
      const int qx0 = uc.q0 + 128 * (int)rank;
      const int row = qx0 + r;
      const size_t bh = (size_t)uc.b * p.Hq + uc.h + x;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        ok = mbar_wait(bar_s_full + 8 * x, s_cnt & 1, 69);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        float s[4][32];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tw + s_col + 32 * c4, s[c4]);
        tmem_wait_ld();
        const int kv0 = j * C::BN;
        if (kv0 + C::BN > p.Lk || (p.causal && kv0 + C::BN - 1 > qx0 + off)) {
          int lim = p.Lk - 1;
          if (p.causal) lim = min(lim, row + off);
          const int rem = lim - kv0;  // may be negative: the whole tile is masked for this row
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * c4 + e > rem) s[c4][e] = -INFINITY;
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            mx0 = fmax3(mx0, s[c4][e], s[c4][e + 1]);
            mx1 = fmax3(mx1, s[c4][e + 2], s[c4][e + 3]);
          }
        const float m_tile = fmaxf(mx0, mx1) * c2;
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_used = m_tile;
        } else if (m_tile > m_used + kRescaleLog2) {
          alpha = ex2_approx(m_used - m_tile);
          m_used = m_tile;
          rescale = true;
        }
        const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
        l *= alpha;
        const uint64_t c2x2 = f2_pack(c2, c2), nm2 = f2_pack(-m_ref, -m_ref);
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t xv = ffma2(f2_pack(s[q4][2 * e], s[q4][2 * e + 1]), c2x2, nm2);
            float p0, p1;
            if (kExp2EmulateMask<C::D> & (1u << e)) {
              f2_unpack(exp2_poly2(xv), p0, p1);
            } else {
              float x0, x1;
              f2_unpack(xv, x0, x1);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            if (e & 1) acc1 = fadd2(acc1, f2_pack(p0, p1));
            else acc0 = fadd2(acc0, f2_pack(p0, p1));
            pk[e] = E::pack2(p0, p1);
          }
          tmem_st16u(tw + s_col + 16 * q4, pk);
        }
        float a0, a1, b0, b1;
        f2_unpack(acc0, a0, a1);
        f2_unpack(acc1, b0, b1);
        l += (a0 + a1) + (b0 + b1);
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c4 = 0; c4 < C::D / 32; ++c4) {
            float o[32];
            tmem_ld32(tw + o_col + 32 * c4, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tw + o_col + 32 * c4, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        if (rank == 0) mbar_arrive(p_full_l);
        else mbar_arrive_cluster(p_full_c);
      }
      if (!ok) break;
      ok = mbar_wait(bar_o_ready + 8 * x, o_cnt & 1, 70);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++o_cnt;
      tc_fence_after();
      const float inv_l = 1.f / l;  // every row sees key 0 in its first tile, so l > 0
      const bool in_range = row < p.Lq;
      uint16_t* orow = p.o + (bh * p.Lq + (in_range ? row : 0)) * C::D;
#pragma unroll
      for (int c4 = 0; c4 < C::D / 32; ++c4) {
        float o[32];
        tmem_ld32(tw + o_col + 32 * c4, o);
        tmem_wait_ld();
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c4);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(E::pack2(o[8 * q + 0] * inv_l, o[8 * q + 1] * inv_l),
                                E::pack2(o[8 * q + 2] * inv_l, o[8 * q + 3] * inv_l),
                                E::pack2(o[8 * q + 4] * inv_l, o[8 * q + 5] * inv_l),
                                E::pack2(o[8 * q + 6] * inv_l, o[8 * q + 7] * inv_l));
        }
      }
      if (in_range && p.lse != nullptr) p.lse[bh * p.Lq + row] = (m_used + log2f(l)) * kLn2;
      tc_fence_before();
      if (rank == 0) mbar_arrive(o_free_l);
      else mbar_arrive_cluster(o_free_c);
    }
  }

  __syncthreads();
  cluster_sync_all();  // no product of the pair is still writing this CTA's TMEM
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
