// prefill.cuh -- forward (prefill) attention on sm_100a: TMA tile loads into a shared-memory
// ring, tcgen05.mma for S = Q.K^T and O += P.V with fp32 accumulators in tensor memory, and a
// running-max / running-sum softmax with one query row per thread.
//
// The tiled, on-chip evaluation follows "Activar Flash Attention con llama.cpp" (section
// "Que es Flash Attention": iterate over blocks in fast on-chip memory instead of storing the
// big intermediates in HBM); the arithmetic is the standard flow S = Q.K^T, P = softmax(S),
// O = P.V of the FlashMLA-ETAP summary ("Mecanismo Central", item 1).
//
// One CTA computes one 128-row query tile of one (batch, head):
//   warps 0-3  softmax: thread r owns query row r of the tile (TMEM lane r); reads S from
//              TMEM, masks, updates the running max / sum, writes P (bf16) into a swizzled
//              shared-memory tile, rescales its O row in TMEM when the max grew a lot, and
//              finally normalises O and stores O and LSE;
//   warp 4     TMA producer: Q once, then K_0, K_1, V_0, K_2, V_1, ... through an NS-stage ring;
//   warp 5     TMEM allocator and MMA issuer (one thread): S_j into one of two TMEM buffers
//              while the softmax works on S_{j-1}, then O += P_{j-1}.V_{j-1}.
// Lazy rescaling: the running max used for the exponent only moves when a tile's max exceeds
// it by more than kRescaleLog2 (log2 units); the final O / l is unchanged by the choice of the
// reference, and p <= 2^kRescaleLog2 stays well inside fp32 / bf16 range.
#pragma once

#include "sm100.cuh"

namespace attn {

struct PrefillParams {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, Lq, Lk, G;
  int n_qtiles;
  int causal;
  float scale_log2;  // scale * log2(e)
};

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;  // query rows per CTA
  static constexpr int BN = 128;  // keys per tile
  static constexpr int DC = D / 64;  // 64-column (128-byte) chunks per row
  static constexpr int CHUNK = 128 * 128;  // one 128-row x 128-byte chunk
  static constexpr int Q_BYTES = DC * CHUNK;
  static constexpr int KV_BYTES = DC * CHUNK;  // one K or V tile
  static constexpr int NS = (D == 128) ? 3 : 4;
  static constexpr int P_BYTES = 2 * CHUNK;  // 128 rows x 128 keys bf16
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;
  static constexpr int OFF_P = OFF_KV + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  // barriers: q_full, kv_full[NS], kv_empty[NS], s_full[2], p_full[2], pv_done[2], drain
  static constexpr int N_BARS = 1 + 2 * NS + 2 + 2 + 2 + 1;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;    // S buffers at columns 0 and 128
  static constexpr uint32_t O_COL = 256;  // O accumulator (D columns)
  static constexpr int THREADS = 192;
};

template <int D>
__global__ void __launch_bounds__(PrefillCfg<D>::THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: heaviest query tiles first; sibling query heads of a kv head adjacent ----
  const int BH = p.B * p.Hq;
  const int qt = p.n_qtiles - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int hkv = h / p.G;
  const int q0 = qt * C::BM;
  const int off = p.Lk - p.Lq;  // bottom-right causal offset
  int n_kv = (p.Lk + C::BN - 1) / C::BN;
  if (p.causal) {
    const int last_row = min(q0 + C::BM - 1, p.Lq - 1);
    n_kv = min(n_kv, (last_row + off) / C::BN + 1);
  }

  const uint32_t bar_q = base + C::OFF_BAR;
  const uint32_t bar_kv_full = bar_q + 8;
  const uint32_t bar_kv_empty = bar_kv_full + 8 * C::NS;
  const uint32_t bar_s_full = bar_kv_empty + 8 * C::NS;
  const uint32_t bar_p_full = bar_s_full + 16;
  const uint32_t bar_pv_done = bar_p_full + 16;
  const uint32_t bar_drain = bar_pv_done + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_kv_full + 8 * s, 1);
      mbar_init(bar_kv_empty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + 8 * i, 1);
      mbar_init(bar_p_full + 8 * i, 128);
      mbar_init(bar_pv_done + 8 * i, 1);
    }
    mbar_init(bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 4) {
    // ------------------------------- TMA producer -------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int zq = b * p.Hq + h, zkv = b * p.Hkv + hkv;
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::DC; ++c) tma_load_3d(base + C::OFF_Q + c * C::CHUNK, &tm_q, bar_q, 64 * c, q0, zq);
      int t = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* m, int tile) {
        const int s = t % C::NS;
        if (t >= C::NS) ok = mbar_wait(bar_kv_empty + 8 * s, ((t / C::NS) & 1) ^ 1, 1);
        if (!ok) return;
        const uint32_t full = bar_kv_full + 8 * s;
        mbar_arrive_expect_tx(full, C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::DC; ++c)
          tma_load_3d(base + C::OFF_KV + s * C::KV_BYTES + c * C::CHUNK, m, full, 64 * c, tile * C::BN, zkv);
        ++t;
      };
      load(&tm_k, 0);
      for (int j = 1; j < n_kv && ok; ++j) {
        load(&tm_k, j);
        if (ok) load(&tm_v, j - 1);
      }
      if (ok) load(&tm_v, n_kv - 1);
      if (!ok) {
        // wait (bounded) for the copies still in flight before the CTA may exit
        mbar_wait_drain(bar_q, 0);
        for (int u = max(0, t - C::NS); u < t; ++u) mbar_wait_drain(bar_kv_full + 8 * (u % C::NS), (u / C::NS) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------- MMA issuer -------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(C::BM, C::BN, false, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(C::BM, D, false, true);
      bool ok = mbar_wait(bar_q, 0, 2);
      bool issued = false;
      int t = 0;
      auto pv = [&](int jj) {
        ok = mbar_wait(bar_p_full + 8 * (jj & 1), (jj >> 1) & 1, 3);
        if (!ok) return;
        const int s = t % C::NS;
        ok = mbar_wait(bar_kv_full + 8 * s, (t / C::NS) & 1, 4);
        if (!ok) return;
        tc_fence_after();
        const uint32_t vb = base + C::OFF_KV + s * C::KV_BYTES;
        const uint32_t pb = base + C::OFF_P + (jj & 1) * C::P_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t ad = make_sdesc(pb + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = make_sdesc(vb + kk * 2048, C::CHUNK, 1024, kSwizzle128B);
          mma_ss(tmem + C::O_COL, ad, bd, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_kv_empty + 8 * s);
        mma_commit(bar_pv_done + 8 * (jj & 1));
        ++t;
      };
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = t % C::NS;
        ok = mbar_wait(bar_kv_full + 8 * s, (t / C::NS) & 1, 5);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb = base + C::OFF_KV + s * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = make_sdesc(base + C::OFF_Q + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = make_sdesc(kb + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024, kSwizzle128B);
          mma_ss(tmem + C::S_COL + (j & 1) * C::BN, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        issued = true;
        mma_commit(bar_s_full + 8 * (j & 1));
        mma_commit(bar_kv_empty + 8 * s);
        ++t;
        if (j > 0) pv(j - 1);
      }
      if (ok) pv(n_kv - 1);
      if (!ok && issued) {
        mma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // ------------------------------- softmax (warps 0-3) -------------------------------
    const int r = threadIdx.x;  // row of the tile == TMEM lane
    const int row = q0 + r;
    const uint32_t tw = tmem + ((uint32_t)(warp * 32) << 16);
    const float c2 = p.scale_log2;
    const int lim_causal = row + off;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = mbar_wait(bar_s_full + 8 * (j & 1), (j >> 1) & 1, 6);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[4][32];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tw + C::S_COL + (j & 1) * C::BN + 32 * c4, s[c4]);
      tmem_wait_ld();
      const int kv0 = j * C::BN;
      if (kv0 + C::BN > p.Lk || (p.causal && kv0 + C::BN - 1 > q0 + off)) {
        int lim = p.Lk - 1;
        if (p.causal) lim = min(lim, lim_causal);
        const int rem = lim - kv0;  // keys c <= rem are visible
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (32 * c4 + e > rem) s[c4][e] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, s[c4][e]);
      const float m_tile = mx * c2;
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
      // P buffer (j & 1) is free once P_{j-2}.V_{j-2} has completed
      if (j >= 2) {
        ok = mbar_wait(bar_pv_done + 8 * (j & 1), ((j - 2) >> 1) & 1, 7);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      float sum = 0.f;
      uint8_t* pbuf = smem + C::OFF_P + (j & 1) * C::P_BYTES;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {  // 8 keys per 16-byte unit
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = ex2_approx(fmaf(s[c4][8 * u2 + 2 * e], c2, -m_ref));
            const float x1 = ex2_approx(fmaf(s[c4][8 * u2 + 2 * e + 1], c2, -m_ref));
            sum += x0 + x1;
            w[e] = pack_bf16x2(x0, x1);
          }
          const int key = 32 * c4 + 8 * u2;  // first key of this unit within the tile
          const int ch = key >> 6, u = (key & 63) >> 3;
          *reinterpret_cast<uint4*>(pbuf + ch * C::CHUNK + swz128_offset((uint32_t)r, (uint32_t)u)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      l += sum;
      if (__any_sync(0xffffffffu, rescale)) {
        // O row must not be touched while P_{j-1}.V_{j-1} is still accumulating into it
        ok = mbar_wait(bar_pv_done + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1, 8);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          float o[32];
          tmem_ld32(tw + C::O_COL + 32 * c4, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tw + C::O_COL + 32 * c4, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p_full + 8 * (j & 1));
    }
    if (ok) {
      ok = mbar_wait(bar_pv_done + 8 * ((n_kv - 1) & 1), ((n_kv - 1) >> 1) & 1, 9);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool in_range = row < p.Lq;
      __nv_bfloat16* orow = p.o + ((size_t)(b * p.Hq + h) * p.Lq + (in_range ? row : 0)) * D;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float o[32];
        tmem_ld32(tw + C::O_COL + 32 * c4, o);
        tmem_wait_ld();
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c4);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[u] = make_uint4(pack_bf16x2(o[8 * u + 0] * inv_l, o[8 * u + 1] * inv_l),
                                pack_bf16x2(o[8 * u + 2] * inv_l, o[8 * u + 3] * inv_l),
                                pack_bf16x2(o[8 * u + 4] * inv_l, o[8 * u + 5] * inv_l),
                                pack_bf16x2(o[8 * u + 6] * inv_l, o[8 * u + 7] * inv_l));
        }
      }
      if (in_range && p.lse != nullptr)
        p.lse[(size_t)(b * p.Hq + h) * p.Lq + row] = (m_used + log2f(l)) * kLn2;
    }
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
