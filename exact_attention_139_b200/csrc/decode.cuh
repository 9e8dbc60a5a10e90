// decode.cuh -- split-KV decode attention (few query tokens, long KV cache) on sm_100a.
//
// A CTA computes, for the R = (Hq/Hkv)*Lq query rows that share a kv head, a partial O over a
// range of that head's keys (fp32, divided by its own softmax sum) and the range's LSE (natural
// log; -inf when no key of the range is visible). The log-sum-exp combine (combine.cuh) merges
// the partials. Ranges are equal chunks of every (batch, kv head) ("split mode"), or, for the
// queries-on-M kernel with no split count given, equal runs of the flattened (batch * Hkv + kv
// head, key) sequence with one CTA per SM slot ("balanced mode", DecodeParams::bal_w).
//
// Three kernels:
//   decode_cc_kernel      fp32 CUDA-core dot products; any supported shape; the baseline.
//   decode_tc_kernel      tcgen05 with the key length on the MMA M dimension: the transposed
//                         flow S^T = K.Q^T, P^T = softmax(S^T), O^T = V^T.P^T of the FlashMLA-ETAP
//                         summary ("Mecanismo Central", items 1-3). With only R = 32 query rows
//                         per kv head, putting keys (64 per tile) on M and queries on N avoids
//                         padding the query dimension to the MMA's minimum M.
//   decode_tn_kernel      tcgen05 with the query rows on M (padded to 64) and keys on N: every
//                         softmax reduction stays inside one thread; the default.
// Latent KV (MLA): V is the first dv columns of each K row; each row is read from HBM once and
// the same shared-memory tile feeds both products. Dense V (GQA decode) streams beside K.
#pragma once

#include "sm100.cuh"

namespace attn {

struct DecodeParams {
  const uint16_t* q;  // 16-bit floats of the kernel's element type
  const uint16_t* k;
  const uint16_t* v;
  float* o_part;    // [num_splits, rows_total, dv]
  float* lse_part;  // [num_splits, rows_total]
  long long rows_total;
  int B, Hq, Hkv, Lq, Lk, d, dv, ldv, G, R;
  int causal;
  int chunk;  // keys per split (multiple of 64)
  int v_is_k;
  float scale_log2;
  // Balanced schedule (queries-on-M kernel, bal_w > 0): CTA c takes keys [c * bal_w, (c + 1) *
  // bal_w) of the flattened (unit, key) space, unit = batch * Hkv + kv head, bal_total = units * Lk
  // keys in all; bal_w <= Lk, so a CTA covers at most two units. Its part of unit u goes to
  // partial slot c - first_cta(u), first_cta(u) = (u * Lk) / bal_w.
  int bal_w;
  long long bal_total;
};

// One contiguous key range of one unit processed by a CTA, and the partial slot it fills.
struct DecodeSeg {
  int unit, j_begin, j_end, piece;
};

// The segments of this CTA: one (split mode: split blockIdx.x of unit blockIdx.y, possibly
// empty) or up to two (balanced mode).
__device__ __forceinline__ int decode_segments(const DecodeParams& p, DecodeSeg (&seg)[2]) {
  if (p.bal_w == 0) {
    const int jb = blockIdx.x * p.chunk;
    seg[0] = DecodeSeg{(int)blockIdx.y, jb, min(p.Lk, jb + p.chunk), (int)blockIdx.x};
    return 1;
  }
  const long long pos0 = (long long)blockIdx.x * p.bal_w;
  const long long pos1 = min(p.bal_total, pos0 + p.bal_w);
  int n = 0;
  for (long long pos = pos0; pos < pos1 && n < 2;) {
    const int u = (int)(pos / p.Lk);
    const long long ub = (long long)u * p.Lk;
    const int jb = (int)(pos - ub);
    const int je = (int)min((long long)p.Lk, pos1 - ub);
    seg[n++] = DecodeSeg{u, jb, je, (int)(blockIdx.x - ub / p.bal_w)};
    pos = ub + je;
  }
  return n;
}

// ======================================================================================
// CUDA-core kernel
// ======================================================================================
constexpr int kCcKeys = 32;      // keys per shared-memory chunk
constexpr int kCcThreads = 256;

__host__ __device__ inline int cc_row_stride(int n) { return n + 8; }  // pad rows by 16 bytes

__host__ inline size_t decode_cc_smem_bytes(int R, int d, int dv, bool separate_v) {
  size_t b = (size_t)R * d * 2;                                   // Q (bf16)
  b += (size_t)kCcKeys * cc_row_stride(d) * 2;                    // K chunk
  if (separate_v) b += (size_t)kCcKeys * cc_row_stride(dv) * 2;   // V chunk
  b += (size_t)64 * kCcKeys * 4;                                  // scores / probabilities
  b += 64 * 4 * 2;                                                // alpha, l
  return b;
}

template <int RMAX, int CPT, typename E>
__global__ void __launch_bounds__(kCcThreads)
    decode_cc_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int split = blockIdx.x;
  const int unit = blockIdx.y;
  const int b = unit / p.Hkv, hkv = unit % p.Hkv;
  const int tid = threadIdx.x;
  const int R = p.R;
  const int ks = cc_row_stride(p.d), vs = cc_row_stride(p.dv);
  const bool sep_v = !p.v_is_k;

  uint16_t* Qs = reinterpret_cast<uint16_t*>(smem);
  uint16_t* Ks = Qs + (size_t)R * p.d;
  uint16_t* Vs = Ks + (size_t)kCcKeys * ks;
  float* Ss = reinterpret_cast<float*>(Vs + (sep_v ? (size_t)kCcKeys * vs : 0));
  float* alpha_s = Ss + 64 * kCcKeys;
  float* l_s = alpha_s + 64;

  const long long row0 = ((long long)b * p.Hq + (long long)hkv * p.G) * p.Lq;
  const int j_begin = split * p.chunk;
  const int j_end = min(p.Lk, j_begin + p.chunk);
  const int off = p.Lk - p.Lq;

  // Q rows of this kv head are contiguous: [R, d]
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + row0 * p.d);
    uint4* dst = reinterpret_cast<uint4*>(Qs);
    for (int i = tid; i < R * p.d / 8; i += kCcThreads) dst[i] = src[i];
  }
  float acc[RMAX][CPT];
#pragma unroll
  for (int r = 0; r < RMAX; ++r)
#pragma unroll
    for (int cc = 0; cc < CPT; ++cc) acc[r][cc] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // meaningful in threads tid < R

  const uint16_t* kbase = p.k + ((long long)b * p.Hkv + hkv) * (long long)p.Lk * p.d;
  const uint16_t* vbase = p.v + ((long long)b * p.Hkv + hkv) * (long long)p.Lk * p.ldv;

  for (int kc = j_begin; kc < j_end; kc += kCcKeys) {
    __syncthreads();  // previous chunk fully consumed
    const int nk = min(kCcKeys, j_end - kc);
    for (int i = tid; i < kCcKeys * (p.d / 8); i += kCcThreads) {
      const int jr = i / (p.d / 8), u = i % (p.d / 8);
      uint4 val = make_uint4(0, 0, 0, 0);
      if (jr < nk) val = *reinterpret_cast<const uint4*>(kbase + (long long)(kc + jr) * p.d + 8 * u);
      *reinterpret_cast<uint4*>(Ks + jr * ks + 8 * u) = val;
    }
    if (sep_v) {
      for (int i = tid; i < kCcKeys * (p.dv / 8); i += kCcThreads) {
        const int jr = i / (p.dv / 8), u = i % (p.dv / 8);
        uint4 val = make_uint4(0, 0, 0, 0);
        if (jr < nk) val = *reinterpret_cast<const uint4*>(vbase + (long long)(kc + jr) * p.ldv + 8 * u);
        *reinterpret_cast<uint4*>(Vs + jr * vs + 8 * u) = val;
      }
    }
    __syncthreads();
    // scores: pairs (r, jr)
    for (int idx = tid; idx < R * kCcKeys; idx += kCcThreads) {
      const int r = idx / kCcKeys, jr = idx % kCcKeys;
      const int key = kc + jr;
      const int i = r % p.Lq;
      float sc = -INFINITY;
      if (jr < nk && (!p.causal || key <= i + off)) {
        const uint32_t* qr = reinterpret_cast<const uint32_t*>(Qs + r * p.d);
        const uint32_t* kr = reinterpret_cast<const uint32_t*>(Ks + jr * ks);
        float a0 = 0.f, a1 = 0.f;
        for (int c = 0; c < p.d / 2; ++c) {
          const float2 qf = E::unpack2(qr[c]);
          const float2 kf = E::unpack2(kr[c]);
          a0 = fmaf(qf.x, kf.x, a0);
          a1 = fmaf(qf.y, kf.y, a1);
        }
        sc = a0 + a1;
      }
      Ss[r * kCcKeys + jr] = sc;
    }
    __syncthreads();
    if (tid < R) {
      float mx = -INFINITY;
      for (int jr = 0; jr < kCcKeys; ++jr) mx = fmaxf(mx, Ss[tid * kCcKeys + jr]);
      const float m_tile = mx * p.scale_log2;
      float alpha = 1.f;
      if (m_tile != -INFINITY && (m_run == -INFINITY || m_tile > m_run + kRescaleLog2)) {
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_tile);
        m_run = m_tile;
      }
      float sum = 0.f;
      for (int jr = 0; jr < kCcKeys; ++jr) {
        const float sc = Ss[tid * kCcKeys + jr];
        const float pr = (sc == -INFINITY) ? 0.f : ex2_approx(fmaf(sc, p.scale_log2, -m_run));
        Ss[tid * kCcKeys + jr] = pr;
        sum += pr;
      }
      l_run = l_run * alpha + sum;
      alpha_s[tid] = alpha;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      if (r < R) {
        const float a = alpha_s[r];
#pragma unroll
        for (int cc = 0; cc < CPT; ++cc) acc[r][cc] *= a;
      }
    }
    const uint16_t* Vsrc = sep_v ? Vs : Ks;
    const int vstride = sep_v ? vs : ks;
    for (int jr = 0; jr < nk; ++jr) {
      float vv[CPT];
#pragma unroll
      for (int cc = 0; cc < CPT; ++cc) {
        const int c = tid + cc * kCcThreads;
        vv[cc] = (c < p.dv) ? E::to_float(Vsrc[jr * vstride + c]) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        if (r < R) {
          const float pr = Ss[r * kCcKeys + jr];
#pragma unroll
          for (int cc = 0; cc < CPT; ++cc) acc[r][cc] = fmaf(pr, vv[cc], acc[r][cc]);
        }
      }
    }
  }
  __syncthreads();
  if (tid < R) {
    l_s[tid] = l_run;
    p.lse_part[(long long)split * p.rows_total + row0 + tid] =
        (l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    if (r < R) {
      const float lr = l_s[r];
      const float inv = (lr > 0.f) ? 1.f / lr : 0.f;
      float* dst = p.o_part + ((long long)split * p.rows_total + row0 + r) * p.dv;
#pragma unroll
      for (int cc = 0; cc < CPT; ++cc) {
        const int c = tid + cc * kCcThreads;
        if (c < p.dv) dst[c] = acc[r][cc] * inv;
      }
    }
  }
}

// ======================================================================================
// tcgen05 kernel, key length on the MMA M dimension
// ======================================================================================
template <int DCH, int NB, int NP>
struct DecodeTcCfg {
  static constexpr int BKV = 64;                 // keys per tile (MMA M of S^T)
  static constexpr int KCH = BKV * 128;          // one 64-row x 128-byte chunk
  static constexpr int STAGE = DCH * KCH;        // one K tile (all d columns)
  static constexpr int QCH = NP * 128;           // one NP-row x 128-byte chunk of Q
  static constexpr int PT = NP * BKV * 2;        // P^T tile bf16 (no swizzle, 8x16B cores)
  static constexpr int TROW = NP + 1;            // reduction scratch row stride (floats)
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_Q = OFF_KV + 2 * STAGE;
  static constexpr int OFF_P = OFF_Q + DCH * QCH;
  static constexpr int OFF_T = OFF_P + 2 * PT;
  static constexpr int OFF_FIN = OFF_T + BKV * TROW * 4;
  // barriers: q_full, kv_full[2], kv_empty[2], s_full[2], p_full[2], pv_done[2], drain, group
  static constexpr int OFF_BAR = (OFF_FIN + 3 * NP * 4 + 7) / 8 * 8;
  static constexpr int N_BARS = 13;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;
  static constexpr uint32_t S_COL = 0;            // S^T buffers: columns [0, 2*NP)
  static constexpr uint32_t O_COL = 2 * NP;       // O^T blocks: NB x NP columns
  static constexpr uint32_t TMEM_COLS = (2 * NP + NB * NP) <= 128 ? 128 : ((2 * NP + NB * NP) <= 256 ? 256 : 512);
  static constexpr int THREADS = 192;
  static_assert(NP == 16 || NP == 32, "query rows padded to 16 or 32");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// TMEM load of NP columns (NP = 16 or 32) for the calling warp's 32 lanes.
template <int NP>
__device__ __forceinline__ void tmem_ld_np(uint32_t taddr, float (&v)[32]) {
  if constexpr (NP == 32) {
    tmem_ld32(taddr, v);
  } else {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
#pragma unroll
    for (int i = 16; i < 32; ++i) v[i] = 0.f;
  }
}

template <int NP>
__device__ __forceinline__ void tmem_st_np(uint32_t taddr, const float (&v)[32]) {
  if constexpr (NP == 32) {
    tmem_st32(taddr, v);
  } else {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32"
        " [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
  }
}

template <int DCH, int NB, int NP, typename E>
__global__ void __launch_bounds__(DecodeTcCfg<DCH, NB, NP>::THREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                     const DecodeParams p) {
  using C = DecodeTcCfg<DCH, NB, NP>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int split = blockIdx.x;
  const int unit = blockIdx.y;
  const int b = unit / p.Hkv, hkv = unit % p.Hkv;
  const long long row0 = ((long long)b * p.Hq + (long long)hkv * p.G) * p.Lq;
  const int j_begin = split * p.chunk;
  const int j_end = min(p.Lk, j_begin + p.chunk);
  const int n_tiles = j_end > j_begin ? (j_end - j_begin + C::BKV - 1) / C::BKV : 0;
  const int off = p.Lk - p.Lq;

  const uint32_t bar_q = base + C::OFF_BAR;
  const uint32_t bar_kv_full = bar_q + 8;
  const uint32_t bar_kv_empty = bar_kv_full + 16;
  const uint32_t bar_s_full = bar_kv_empty + 16;
  const uint32_t bar_p_full = bar_s_full + 16;
  const uint32_t bar_pv_done = bar_p_full + 16;
  const uint32_t bar_drain = bar_pv_done + 16;
  const uint32_t bar_grp = bar_drain + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  float* T = reinterpret_cast<float*>(smem + C::OFF_T);
  float* fin_m = reinterpret_cast<float*>(smem + C::OFF_FIN);
  float* fin_a = fin_m + NP;
  float* fin_l = fin_a + NP;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_kv_full + 8 * i, 1);
      mbar_init(bar_kv_empty + 8 * i, 1);
      mbar_init(bar_s_full + 8 * i, 1);
      mbar_init(bar_p_full + 8 * i, 128);
      mbar_init(bar_pv_done + 8 * i, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_grp, 128);
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
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kv);
      mbar_arrive_expect_tx(bar_q, DCH * C::QCH);
#pragma unroll
      for (int c = 0; c < DCH; ++c) tma_load_2d(base + C::OFF_Q + c * C::QCH, &tm_q, bar_q, 64 * c, (int)row0);
      const int z = b * p.Hkv + hkv;
      int t = 0;
      bool ok = true;
      for (; t < n_tiles; ++t) {
        const int s = t & 1;
        if (t >= 2) ok = mbar_wait(bar_kv_empty + 8 * s, ((t >> 1) & 1) ^ 1, 21);
        if (!ok) break;
        const uint32_t full = bar_kv_full + 8 * s;
        mbar_arrive_expect_tx(full, C::STAGE);
#pragma unroll
        for (int c = 0; c < DCH; ++c)
          tma_load_3d(base + C::OFF_KV + s * C::STAGE + c * C::KCH, &tm_kv, full, 64 * c, j_begin + t * C::BKV, z);
      }
      if (!ok) {
        mbar_wait_drain(bar_q, 0);
        for (int u = max(0, t - 2); u < t; ++u) mbar_wait_drain(bar_kv_full + 8 * (u & 1), (u >> 1) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------- MMA issuer -------------------------------
    // warp-uniform control flow and waits; the elected lane issues and commits
    if (n_tiles > 0) {
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_s = make_idesc(64, NP, false, false, E::kFmt);  // S^T = K.Q^T
      constexpr uint32_t idesc_o = make_idesc(128, NP, true, false, E::kFmt);  // O^T += V^T.P^T
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, 22));
      bool issued = false;
      auto pv = [&](int tt) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_p_full + 8 * (tt & 1), (tt >> 1) & 1, 23));
        if (!ok) return;
        tc_fence_after();
        const uint32_t kb = base + C::OFF_KV + (tt & 1) * C::STAGE;
        const uint32_t pb = base + C::OFF_P + (tt & 1) * C::PT;
        if (leader) {
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
            for (int kk = 0; kk < C::BKV / 16; ++kk) {
              // A = V^T block nb: dv rows [128nb, 128nb+128) = chunks 2nb, 2nb+1 (MN-major)
              const uint64_t ad = make_sdesc(kb + (2 * nb) * C::KCH + kk * 2048, C::KCH, 1024, kSwizzle128B);
              // B = P^T: NP x 64 keys, K-major 8x16B core matrices (LBO 128, SBO 1024)
              const uint64_t bd = make_sdesc(pb + kk * 256, 128, 1024, kSwizzleNone);
              mma_ss(tmem + C::O_COL + nb * NP, ad, bd, idesc_o, (tt > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(bar_kv_empty + 8 * (tt & 1));
          mma_commit(bar_pv_done + 8 * (tt & 1));
        }
        __syncwarp();
      };
      for (int t = 0; t < n_tiles && ok; ++t) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_kv_full + 8 * (t & 1), (t >> 1) & 1, 24));
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb = base + C::OFF_KV + (t & 1) * C::STAGE;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4 * DCH; ++kk) {
            const uint64_t ad = make_sdesc(kb + (kk >> 2) * C::KCH + (kk & 3) * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = make_sdesc(base + C::OFF_Q + (kk >> 2) * C::QCH + (kk & 3) * 32, 16, 1024, kSwizzle128B);
            mma_ss(tmem + C::S_COL + (t & 1) * NP, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_s_full + 8 * (t & 1));
        }
        __syncwarp();
        issued = true;
        if (t > 0) pv(t - 1);
      }
      if (ok) pv(n_tiles - 1);
      if (!ok && issued) {
        if (leader) mma_commit(bar_drain);
        __syncwarp();
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // --------------------------- softmax warpgroup (warps 0-3) ---------------------------
    const int tid = threadIdx.x;        // 0..127
    const bool has_row = lane < 16;     // M = 64 layout: keys live in lanes 0-15 of each quadrant
    const int kr = 16 * warp + lane;    // key row of the tile for has_row lanes
    const uint32_t tw = tmem + ((uint32_t)(warp * 32) << 16);
    constexpr int PARTS = 128 / NP;     // threads per query column in the reductions
    constexpr int RPP = C::BKV / PARTS; // key rows per thread in the reductions
    const int col = tid / PARTS, part = tid % PARTS;
    const float c2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;  // of query column `col` (replicated over parts)
    bool ok = true;
    uint32_t gphase = 0;
    // barrier over the 128 softmax threads with a bounded wait (a plain bar.sync cannot give up)
    auto group_sync = [&]() -> bool {
      mbar_arrive(bar_grp);
      const bool r = mbar_wait(bar_grp, gphase, 29);
      gphase ^= 1u;
      return __all_sync(0xffffffffu, r);
    };
    // per-column visibility limit (causal): query column n is token i = n % Lq
    for (int t = 0; t < n_tiles; ++t) {
      ok = mbar_wait(bar_s_full + 8 * (t & 1), (t >> 1) & 1, 25);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float x[32];
      tmem_ld_np<NP>(tw + C::S_COL + (t & 1) * NP, x);
      tmem_wait_ld();
      const int key = j_begin + t * C::BKV + kr;
      if (has_row) {
#pragma unroll
        for (int n = 0; n < NP; ++n) {
          const bool vis = key < j_end && n < p.R && (!p.causal || key <= (n % p.Lq) + off);
          T[kr * C::TROW + n] = vis ? x[n] : -INFINITY;
        }
      }
      ok = group_sync();
      if (!ok) break;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < RPP; ++i) mx = fmaxf(mx, T[(part * RPP + i) * C::TROW + col]);
#pragma unroll
      for (int sh = 1; sh < PARTS; sh <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
      const float m_tile = mx * c2;
      float alpha = 1.f;
      if (m_tile != -INFINITY && (m_run == -INFINITY || m_tile > m_run + kRescaleLog2)) {
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_tile);
        m_run = m_tile;
      }
      if (part == 0) {
        fin_m[col] = m_run;
        fin_a[col] = alpha;
      }
      // P^T buffer (t & 1) is free once O^T += V^T.P^T of tile t-2 has completed
      if (t >= 2) {
        ok = mbar_wait(bar_pv_done + 8 * (t & 1), ((t - 2) >> 1) & 1, 26);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      ok = group_sync();
      if (!ok) break;
      uint8_t* pbuf = smem + C::OFF_P + (t & 1) * C::PT;
      if (has_row) {
#pragma unroll
        for (int n = 0; n < NP; ++n) {
          const float sv = T[kr * C::TROW + n];
          const float mn = fin_m[n];
          const float pr = (sv == -INFINITY) ? 0.f : ex2_approx(fmaf(sv, c2, -mn));
          T[kr * C::TROW + n] = pr;
          // element (n, key kr) of the K-major no-swizzle P^T tile
          const uint32_t o = (uint32_t)(n >> 3) * 1024u + (uint32_t)(kr >> 3) * 128u +
                             (uint32_t)(n & 7) * 16u + (uint32_t)(kr & 7) * 2u;
          *reinterpret_cast<uint16_t*>(pbuf + o) = (uint16_t)(E::pack2(pr, 0.f) & 0xFFFFu);
        }
      }
      ok = group_sync();
      if (!ok) break;
      float sm = 0.f;
#pragma unroll
      for (int i = 0; i < RPP; ++i) sm += T[(part * RPP + i) * C::TROW + col];
#pragma unroll
      for (int sh = 1; sh < PARTS; sh <<= 1) sm += __shfl_xor_sync(0xffffffffu, sm, sh);
      l_run = l_run * alpha + sm;
      bool any_rescale = false;
#pragma unroll
      for (int n = 0; n < NP; ++n) any_rescale |= (fin_a[n] != 1.f);
      if (any_rescale && t > 0) {
        ok = mbar_wait(bar_pv_done + 8 * ((t - 1) & 1), ((t - 1) >> 1) & 1, 27);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float a[32];
#pragma unroll
        for (int n = 0; n < 32; ++n) a[n] = (n < NP) ? fin_a[n] : 1.f;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          float o[32];
          tmem_ld_np<NP>(tw + C::O_COL + nb * NP, o);
          tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < 32; ++n) o[n] *= a[n];
          tmem_st_np<NP>(tw + C::O_COL + nb * NP, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p_full + 8 * (t & 1));
      ok = group_sync();  // T and fin_* are rewritten by the next tile
      if (!ok) break;
    }
    if (ok && n_tiles > 0) {
      ok = mbar_wait(bar_pv_done + 8 * ((n_tiles - 1) & 1), ((n_tiles - 1) >> 1) & 1, 28);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      if (part == 0) {
        fin_l[col] = l_run;
        if (col < p.R)
          p.lse_part[(long long)split * p.rows_total + row0 + col] =
              (l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      }
      ok = group_sync();
    }
    if (ok) {
      tc_fence_after();
      float inv[32];
#pragma unroll
      for (int n = 0; n < 32; ++n) {
        const float ln = (n < NP) ? fin_l[n] : 0.f;
        inv[n] = (ln > 0.f) ? 1.f / ln : 0.f;
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        float o[32];
        if (n_tiles > 0) {
          tmem_ld_np<NP>(tw + C::O_COL + nb * NP, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int n = 0; n < 32; ++n) o[n] = 0.f;
        }
        const int c = 128 * nb + 32 * warp + lane;  // dv column = TMEM lane of the block
#pragma unroll
        for (int n = 0; n < NP; ++n)
          if (n < p.R) p.o_part[((long long)split * p.rows_total + row0 + n) * p.dv + c] = o[n] * inv[n];
      }
    }
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ======================================================================================
// tcgen05 kernel, queries on the MMA M dimension (padded to 64), keys on N
// ======================================================================================
// S = Q.K^T with M = 64 query rows (R <= 32 real rows; rows 32..63 of the A operand read whatever
// follows in shared memory and are never used: MMA rows are independent), N = BK keys, K = d.
// Each softmax thread then owns one query row and reduces over its keys in registers, so a tile
// needs no block-level synchronisation. O = P.V with M = 64, N = dv in pieces of <= 256.
// K/V tiles stream through an NST-stage ring; a stage is released once P.V of its tile is done.
// TMEM (M = 64 layout: row m lives in lane (m % 16) + 32 * (m / 16) of a lane half):
//   lane half 0 (lanes 0-15 of each quadrant): O, columns [0, dv)
//   lane half 1 (lanes 16-31 of each quadrant): S double buffer of NACC partial tiles,
//                columns [(b * NACC + a) * BK, ... + BK) for buffer b, partial a
// Warps: 0-1 softmax (lanes 16-31 hold S rows, lanes 0-15 the matching O rows), 2 TMA producer,
// 3 TMEM allocator + P.V issuer, 4 .. 3 + NACC S issuers.
template <int DCH, int NPIECE, int BK, int NST, bool SEPV>
struct DecodeTnCfg {
  // SEPV: V is a separate dense tensor (dv == d); each ring stage then holds the K tile followed
  // by the V tile. Otherwise V is the first dv columns of the latent K tile.
  // S = Q.K^T is accumulated in NACC independent TMEM tiles (chunk c of the d columns goes to
  // tile c % NACC) issued interleaved: back-to-back MMAs into one accumulator serialise on its
  // latency, independent ones overlap. The softmax adds the partial tiles.
  static constexpr int NACC = (DCH % 3 == 0) ? 3 : ((DCH % 2 == 0) ? 2 : 1);
  static constexpr int KCH = BK * 128;           // one BK-key x 128-byte chunk
  static constexpr int VOFF = DCH * KCH;         // offset of the V tile inside a stage (SEPV)
  static constexpr int STAGE = (SEPV ? 2 : 1) * DCH * KCH;
  static constexpr int QCH = 32 * 128;           // 32 query rows x 128 bytes
  static constexpr int PB = 32 * 128;            // P tile: 32 rows x (<= 64) keys bf16, 128-B rows
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_Q = OFF_KV + NST * STAGE;
  static constexpr int OFF_P = OFF_Q + DCH * QCH;   // right after Q: rows 32..63 of the M=64 reads
  static constexpr int OFF_PAD = OFF_P + 2 * PB;    // 4 KB of slack read as rows 32..63 of P1
  static constexpr int OFF_BAR = OFF_PAD + 4096;
  // barriers: q_full, kv_full[NST], kv_empty[NST], s_full[2], p_full[2], pv_done[2],
  // drain[1 + NACC] (one per MMA-issuing warp), q_empty, o_free
  static constexpr int N_BARS = 1 + 2 * NST + 6 + 1 + NACC + 2;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t S_LANE = 16;
  // warps: 0-1 softmax, 2 TMA producer, 3 TMEM allocator + P.V issuer, 4.. S issuers (one per
  // partial accumulator): one thread issuing tcgen05.mma back to back is limited by its own
  // instruction latency for these small shapes, so the S products are spread over NACC warps.
  static constexpr int THREADS = 32 * (4 + NACC);
  static_assert(BK == 32 || BK == 48 || BK == 64, "key tile");
  static_assert(2 * NACC * BK <= 512, "S partial tiles fit in one lane half");
  static_assert(OFF_Q % 1024 == 0 && KCH % 1024 == 0, "128-byte swizzle atoms need 1 KB alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Load BK (32, 48 or 64) fp32 columns of the calling warp's lanes from TMEM.
template <int BK>
__device__ __forceinline__ void tmem_ld_keys(uint32_t taddr, float (&x)[64]) {
  float a[32];
  tmem_ld32(taddr, a);
#pragma unroll
  for (int e = 0; e < 32; ++e) x[e] = a[e];
  if constexpr (BK == 64) {
    float b[32];
    tmem_ld32(taddr + 32, b);
#pragma unroll
    for (int e = 0; e < 32; ++e) x[32 + e] = b[e];
  } else if constexpr (BK == 48) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr + 32));
#pragma unroll
    for (int e = 0; e < 16; ++e) x[32 + e] = __uint_as_float(r[e]);
  }
}

template <int DCH, int NPIECE, int BK, int NST, bool SEPV, typename E>
__global__ void __launch_bounds__(DecodeTnCfg<DCH, NPIECE, BK, NST, SEPV>::THREADS, 1)
    decode_tn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using C = DecodeTnCfg<DCH, NPIECE, BK, NST, SEPV>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  DecodeSeg seg[2];
  const int nseg = decode_segments(p, seg);
  auto seg_tiles = [&](int g) {
    return seg[g].j_end > seg[g].j_begin ? (seg[g].j_end - seg[g].j_begin + BK - 1) / BK : 0;
  };
  auto seg_row0 = [&](int g) {
    const int b = seg[g].unit / p.Hkv, hkv = seg[g].unit % p.Hkv;
    return ((long long)b * p.Hq + (long long)hkv * p.G) * p.Lq;
  };
  const int off = p.Lk - p.Lq;
  const int NW = p.dv / NPIECE;  // columns per O piece (multiple of 64)
  // TMEM columns: O needs dv (lane half 0), the S partial tiles 2 * NACC * BK (lane half 1)
  const int cols_needed = max(p.dv, 2 * C::NACC * BK);
  const uint32_t TMEM_COLS = cols_needed <= 128 ? 128u : (cols_needed <= 256 ? 256u : 512u);

  const uint32_t bar_q = base + C::OFF_BAR;
  const uint32_t bar_kv_full = bar_q + 8;
  const uint32_t bar_kv_empty = bar_kv_full + 8 * NST;
  const uint32_t bar_s_full = bar_kv_empty + 8 * NST;
  const uint32_t bar_p_full = bar_s_full + 16;
  const uint32_t bar_pv_done = bar_p_full + 16;
  const uint32_t bar_drain = bar_pv_done + 16;
  const uint32_t bar_q_empty = bar_drain + 8 * (1 + C::NACC);  // all S of a segment issued and done
  const uint32_t bar_o_free = bar_q_empty + 8;                 // the softmax has read O out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(bar_kv_full + 8 * i, 1);
      mbar_init(bar_kv_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + 8 * i, C::NACC);  // one commit per S issuer
      mbar_init(bar_p_full + 8 * i, 64);
      mbar_init(bar_pv_done + 8 * i, 1);
    }
    for (int i = 0; i <= C::NACC; ++i) mbar_init(bar_drain + 8 * i, 1);
    mbar_init(bar_q_empty, C::NACC);
    mbar_init(bar_o_free, 64);
    fence_mbar_init();
  }
  if (warp == 3) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 2) {
    // ------------------------------- TMA producer -------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kv);
      if constexpr (SEPV) tma_prefetch_desc(&tm_v);
      int t = 0, qn = 0;  // tiles and Q tiles loaded so far
      bool ok = true;
      for (int g = 0; g < nseg && ok; ++g) {
        const int n_tiles = seg_tiles(g);
        if (n_tiles == 0) continue;
        // Q of this segment's unit, once every S product of the previous segment is done
        if (qn > 0) ok = mbar_wait(bar_q_empty, (qn - 1) & 1, 40);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_q, DCH * C::QCH);
#pragma unroll
        for (int c = 0; c < DCH; ++c) tma_load_2d(base + C::OFF_Q + c * C::QCH, &tm_q, bar_q, 64 * c, (int)seg_row0(g));
        ++qn;
        const int z = seg[g].unit;
        for (int tt = 0; tt < n_tiles; ++tt, ++t) {
          const int s = t % NST;
          if (t >= NST) ok = mbar_wait(bar_kv_empty + 8 * s, ((t / NST) & 1) ^ 1, 41);
          if (!ok) break;
          const uint32_t full = bar_kv_full + 8 * s;
          const int j = seg[g].j_begin + tt * BK;
          mbar_arrive_expect_tx(full, C::STAGE);
#pragma unroll
          for (int c = 0; c < DCH; ++c)
            tma_load_3d(base + C::OFF_KV + s * C::STAGE + c * C::KCH, &tm_kv, full, 64 * c, j, z);
          if constexpr (SEPV) {
#pragma unroll
            for (int c = 0; c < DCH; ++c)
              tma_load_3d(base + C::OFF_KV + s * C::STAGE + C::VOFF + c * C::KCH, &tm_v, full, 64 * c, j, z);
          }
        }
      }
      if (!ok) {
        if (qn > 0) mbar_wait_drain(bar_q, (qn - 1) & 1);
        for (int u = max(0, t - NST); u < t; ++u) mbar_wait_drain(bar_kv_full + 8 * (u % NST), (u / NST) & 1);
      }
    }
  } else if (warp >= 4) {
    // -------------------- S issuers: partial a = chunks a, a + NACC, ... --------------------
    // Each issuing warp runs its control flow and waits warp-uniformly; its elected lane issues
    // the products and commits (issuing from inside a one-lane branch is measurably slower).
    {
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_s = make_idesc(64, BK, false, false, E::kFmt);  // S = Q.K^T
      const int a = warp - 4;
      const uint32_t s_tmem = tmem + (C::S_LANE << 16) + C::S_COL + a * BK;
      const uint64_t qdesc = make_sdesc(base + C::OFF_Q + a * C::QCH, 16, 1024, kSwizzle128B);
      bool ok = true, issued = false;
      int t = 0, qn = 0;
      for (int g = 0; g < nseg && ok; ++g) {
        const int n_tiles = seg_tiles(g);
        if (n_tiles == 0) continue;
        ok = __all_sync(0xffffffffu, mbar_wait(bar_q, qn & 1, 42));
        if (!ok) break;
        ++qn;
        for (int tt = 0; tt < n_tiles && ok; ++tt, ++t) {
          ok = mbar_wait(bar_kv_full + 8 * (t % NST), (t / NST) & 1, 44);
          // S buffer (t & 1) was last read by the softmax of tile t - 2
          if (ok && t >= 2) ok = mbar_wait(bar_p_full + 8 * (t & 1), ((t - 2) >> 1) & 1, 50);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const uint64_t kdesc = make_sdesc(base + C::OFF_KV + (t % NST) * C::STAGE + a * C::KCH, 16, 1024, kSwizzle128B);
          const uint32_t d = s_tmem + (t & 1) * C::NACC * BK;
          if (leader) {
#pragma unroll
            for (int i = 0; i < DCH / C::NACC; ++i) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                // descriptor start addresses advance by whole 16-byte units
                const uint64_t qa = qdesc + (uint64_t)((i * C::NACC * C::QCH + ks * 32) >> 4);
                const uint64_t kb = kdesc + (uint64_t)((i * C::NACC * C::KCH + ks * 32) >> 4);
                mma_ss(d, qa, kb, idesc_s, (i > 0 || ks > 0) ? 1u : 0u);
              }
            }
            mma_commit(bar_s_full + 8 * (t & 1));
          }
          __syncwarp();
          issued = true;
        }
        if (!ok) break;
        if (leader) mma_commit(bar_q_empty);  // this segment's Q may be replaced once these products are done
        __syncwarp();
      }
      if (!ok && issued) {
        if (leader) mma_commit(bar_drain + 8 * (1 + a));
        __syncwarp();
        mbar_wait_drain(bar_drain + 8 * (1 + a), 0);
      }
    }
  } else if (warp == 3) {
    // ------------------------------- P.V issuer -------------------------------
    {
      const bool leader = elect_one_sync();
      const uint32_t idesc_o = make_idesc(64, NW, false, true, E::kFmt);  // O += P.V
      bool ok = true, issued = false;
      int t = 0, segs_done = 0;
      for (int g = 0; g < nseg && ok; ++g) {
        const int n_tiles = seg_tiles(g);
        if (n_tiles == 0) continue;
        // the first product of a segment overwrites O: the previous segment's O must be read out
        if (segs_done > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_o_free, (segs_done - 1) & 1, 39));
        if (!ok) break;
        for (int tt = 0; tt < n_tiles && ok; ++tt, ++t) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_p_full + 8 * (t & 1), (t >> 1) & 1, 43));
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = base + C::OFF_KV + (t % NST) * C::STAGE + (SEPV ? C::VOFF : 0);  // V rows
          const uint32_t pb = base + C::OFF_P + (t & 1) * C::PB;
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = make_sdesc(pb + kk * 32, 16, 1024, kSwizzle128B);
#pragma unroll
              for (int h = 0; h < NPIECE; ++h) {
                // B = V rows of this tile, dv columns [h*NW, h*NW + NW): MN-major, 64-column atoms
                const uint64_t bd = make_sdesc(kb + (h * NW / 64) * C::KCH + kk * 2048, C::KCH, 1024, kSwizzle128B);
                mma_ss(tmem + h * NW, ad, bd, idesc_o, (tt > 0 || kk > 0) ? 1u : 0u);
              }
            }
            // the S products of this tile completed before its softmax started, so this commit
            // also covers every read of the stage
            mma_commit(bar_kv_empty + 8 * (t % NST));
            mma_commit(bar_pv_done + 8 * (t & 1));
          }
          __syncwarp();
          issued = true;
        }
        ++segs_done;
      }
      if (!ok && issued) {
        if (leader) mma_commit(bar_drain);
        __syncwarp();
        mbar_wait_drain(bar_drain, 0);
      }
    }
  } else {
    // --------------------------- softmax warps 0-1 ---------------------------
    const bool s_lane = lane >= 16;
    const int m = 16 * warp + (lane & 15);  // query row (S row for lanes 16-31, O row for 0-15)
    const bool row_ok = m < p.R;
    const int qi = m % p.Lq;
    const uint32_t tw = tmem + ((uint32_t)(warp * 32) << 16);
    const float c2 = p.scale_log2;
    bool ok = true;
    int t = 0;
    for (int g = 0; g < nseg && ok; ++g) {
      const int n_tiles = seg_tiles(g);
      const int j_begin = seg[g].j_begin, j_end = seg[g].j_end;
      float m_run = -INFINITY, l_run = 0.f;
      for (int tt = 0; tt < n_tiles; ++tt, ++t) {
        ok = mbar_wait(bar_s_full + 8 * (t & 1), (t >> 1) & 1, 45);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float x[64];
        tmem_ld_keys<BK>(tw + C::S_COL + (t & 1) * C::NACC * BK, x);
#pragma unroll
        for (int a = 1; a < C::NACC; ++a) {
          float y[64];
          tmem_ld_keys<BK>(tw + C::S_COL + ((t & 1) * C::NACC + a) * BK, y);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < BK; ++e) x[e] += y[e];
        }
        tmem_wait_ld();
        const int k0 = j_begin + tt * BK;
        int lim = j_end - 1;
        if (p.causal) lim = min(lim, qi + off);
        const int rem = lim - k0;  // keys c <= rem of this tile are visible
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < BK; ++e) {
          if (e > rem) x[e] = -INFINITY;
          mx = fmaxf(mx, x[e]);
        }
        const float m_tile = mx * c2;
        float alpha = 1.f;
        if (m_tile != -INFINITY) {
          if (m_run == -INFINITY) {
            m_run = m_tile;  // O row and l are still zero: nothing to rescale
          } else if (m_tile > m_run + kRescaleLog2) {
            alpha = ex2_approx(m_run - m_tile);
            m_run = m_tile;
          }
        }
        const float m_ref = (m_run == -INFINITY) ? 0.f : m_run;
        // P buffer (t & 1) is free once P.V of tile t-2 has completed
        if (t >= 2) {
          ok = mbar_wait(bar_pv_done + 8 * (t & 1), ((t - 2) >> 1) & 1, 46);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        float sum = 0.f;
        uint8_t* prow = smem + C::OFF_P + (t & 1) * C::PB;
#pragma unroll
        for (int u = 0; u < BK / 8; ++u) {  // 8 keys per 16-byte unit
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2_approx(fmaf(x[8 * u + 2 * e], c2, -m_ref));
            const float p1 = ex2_approx(fmaf(x[8 * u + 2 * e + 1], c2, -m_ref));
            sum += p0 + p1;
            w4[e] = E::pack2(p0, p1);
          }
          if (s_lane)
            *reinterpret_cast<uint4*>(prow + swz128_offset((uint32_t)m, (uint32_t)u)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        l_run = l_run * alpha + sum;
        // rescale the O rows whose reference moved (rare): lanes 0-15 own those O rows
        const float alpha_o = __shfl_down_sync(0xffffffffu, alpha, 16);
        const bool need = tt > 0 && __any_sync(0xffffffffu, s_lane && alpha != 1.f);
        if (need) {
          // O is stable once P.V of tile t-1 is done; S of tile t+1 (same columns, other lane
          // half, rewritten unchanged below) must have landed too, whichever segment it is in
          const bool next_tile = tt + 1 < n_tiles || (g + 1 < nseg && seg_tiles(g + 1) > 0);
          ok = mbar_wait(bar_pv_done + 8 * ((t - 1) & 1), ((t - 1) >> 1) & 1, 47);
          if (ok && next_tile) ok = mbar_wait(bar_s_full + 8 * ((t + 1) & 1), ((t + 1) >> 1) & 1, 48);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const float sc = s_lane ? 1.f : alpha_o;
          for (int cg = 0; cg < p.dv / 32; ++cg) {
            float o[32];
            tmem_ld32(tw + 32 * cg, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= sc;
            tmem_st32(tw + 32 * cg, o);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_p_full + 8 * (t & 1));
      }
      if (!ok) break;
      if (n_tiles > 0) {
        ok = mbar_wait(bar_pv_done + 8 * ((t - 1) & 1), ((t - 1) >> 1) & 1, 49);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      // lanes 16-31 hold (m_run, l_run) of row m; lanes 0-15 hold O row m
      const long long row0 = seg_row0(g);
      const int piece = seg[g].piece;
      const float l_o = __shfl_down_sync(0xffffffffu, l_run, 16);
      if (s_lane && row_ok)
        p.lse_part[(long long)piece * p.rows_total + row0 + m] = (l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      const float inv = (l_o > 0.f) ? 1.f / l_o : 0.f;
      float* dst = p.o_part + ((long long)piece * p.rows_total + row0 + m) * p.dv;
      tc_fence_after();
      for (int cg = 0; cg < p.dv / 32; ++cg) {
        float o[32];
        if (n_tiles > 0) {
          tmem_ld32(tw + 32 * cg, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0.f;
        }
        if (!s_lane && row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * cg + e) = make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
        }
      }
      // O may now be overwritten by the next segment's first P.V product
      tc_fence_before();
      mbar_arrive(bar_o_free);
    }
  }

  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace attn
