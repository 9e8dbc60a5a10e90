// prefill2.cuh -- persistent forward (prefill) attention on sm_100a with two query tiles per CTA.
//
// Arithmetic: the standard flow S = Q.K^T, P = softmax(S), O = P.V of the FlashMLA-ETAP summary
// ("Mecanismo Central", item 1), evaluated tile by tile in on-chip memory as in "Activar Flash
// Attention con llama.cpp" ("Que es Flash Attention"): TMA tile loads, tcgen05.mma with fp32
// accumulators in TMEM, a running-max / running-sum softmax with one query row per thread, exp2
// with the scale folded in, lazy rescaling (the exponent reference moves only when a tile's max
// exceeds it by more than 2^8), causal tiles above the diagonal never loaded.
//
// Organisation, chosen so the tensor core rarely waits for the exponentials:
//   * a work unit is a pair of 128-row query tiles (A = rows q0.., B = rows q0+128..) of one
//     (batch, head); both share every K/V tile;
//   * two softmax warpgroups (A: warps 0-3, B: warps 4-7) each own one tile, one query row per
//     thread (TMEM lane); while one computes exponentials the MMA thread issues the other's products:
//         S_A(0) S_B(0) | PV_A(0) S_A(1) | PV_B(0) S_B(1) | PV_A(1) S_A(2) | ...
//     A single issuing thread keeps each tile's products contiguous on the tensor core; issuing
//     A and B from two warps interleaved them and was measured slower;
//   * P (16-bit) is written back into TMEM over the S columns it came from, and P.V takes its A
//     operand from TMEM: shared memory holds only Q_A, Q_B and a K/V ring whose stage j holds
//     K_j and V_j, and the tensor core reads half as many operand bytes from shared memory as
//     with P in shared memory (also measured: an SS-operand P.V made the kernel
//     shared-memory-bandwidth bound);
//   * the grid is persistent (one CTA per SM); units are sorted by causal cost inside groups of
//     batches whose K/V fits in half the L2 and dealt boustrophedon (see prefill_unit_index), and
//     every barrier phase carries across units;
//   * the block-sparse instantiation (SPARSE) walks the union of the two tiles' caller-given
//     key-block lists instead of the causal prefix.
//   * the output of a tile is written by a separate epilogue warpgroup (warps 8-11): when a
//     tile's last P is ready, its softmax warpgroup leaves the row statistics in shared memory and
//     moves on to the next unit, while the epilogue warpgroup waits for the last P.V, reads O out
//     of TMEM (releasing it for the next unit's first P.V) and stores it through a staging buffer
//     with TMA. (With the epilogue in the softmax warpgroups the next unit's first P.V waited for
//     the last P.V, the output stores and a softmax in a row.)
// Warps: 0-7 softmax, 8-11 epilogue, 12 TMA producer, 13 TMEM allocator + MMA issuer, 14-15 idle.
// Registers (setmaxnreg): 184 per softmax thread, 64 per epilogue thread, 80 for warps 12-15; at
// launch 128 each (512 threads), and 2 * 184 + 64 + 80 = 4 * 128. (Measured against 176 / 64 / 96:
// fewer spills in the softmax and +0.2 to +2 % on every shape; 184 / 56 / 88 was mixed.)
#pragma once

#include "sm100.cuh"

namespace attn {

struct Prefill2Params {
  uint16_t* o;  // 16-bit floats of the kernel's element type
  float* lse;
  int B, Hq, Hkv, Lq, Lk, G;
  int n_pairs;  // adjacent pairs: ceil(ceil(Lq / 128) / 2)
  int n_units;  // sibling pairs: n_qblocks * B * Hq / 2; adjacent pairs: n_pairs * B * Hq
  int sib;      // 1: the two tiles of a unit are query heads h, h + 1 at the same 128 rows
  int group_b;  // batches per scheduling group (their K/V fits comfortably in L2)
  int causal;
  float scale_log2;
  // block-sparse mode only: per (batch, head, 128-row query block) a sorted list of distinct
  // 128-key blocks; cnt [B, Hq, n_qblocks], idx [B, Hq, n_qblocks, max_blk]
  const int32_t* blk_idx;
  const int32_t* blk_cnt;
  int max_blk, n_qblocks, n_kblocks;
};

// Key pairs e (0..15 within each group of 32 keys) whose exponentials are computed with the FMA
// polynomial (bit e set) instead of ex2.approx on the MUFU unit. Measured on B200 with the
// warp-uniform issuer and the split P hand-off (TFLOP/s; 8K causal / 2K batched / 128K / 8K at
// d = 64): none 1283 / 1053 / 1142 / 722, one pair in sixteen 1293 / 1053 / 1143 / 710, one in
// eight 1228 / 995 / 1077 / 703, one in four 1137 / 960 / 1003 / 664. (With the earlier one-lane
// issuer one in eight had been best: the polynomial's extra instructions now cost more than the
// MUFU time they save.)
#ifndef ATTN_EXP2_EMULATE_MASK
#define ATTN_EXP2_EMULATE_MASK(D) ((D) == 64 ? 0x0000u : 0x0080u)
#endif
template <int D>
constexpr uint32_t kExp2EmulateMask = ATTN_EXP2_EMULATE_MASK(D);

// Shared memory: Q_A and Q_B, then a ring of NS stages, stage j holding K_j and V_j under one
// full and one empty barrier; a stage is released by one commit after the last P.V product of its
// tile. (Measured alternative: separate K and V rings, K three deep and V two deep, each slot
// released after its last reader, so that K is fetched further ahead: same results, 3 % slower
// at 8K and 2K. Cycle counters in the MMA-issuing thread showed that its waits for K and V took
// under 4 % of its time either way: the loads are not what paces the kernel.)
template <int D>
struct Prefill2Cfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int DC = D / 64;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int Q_BYTES = DC * CHUNK;
  static constexpr int KV_BYTES = DC * CHUNK;       // one K or V tile
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;  // ring stage j holds (K_j, V_j)
  static constexpr int NS = (D == 128) ? 2 : 3;
  static constexpr int OFF_Q = 0;  // Q_A, then Q_B
  static constexpr int OFF_KV = 2 * Q_BYTES;
  // Output staging: the epilogue warpgroup writes 64 columns of a tile of O (16-bit, 128-byte
  // swizzled like Q) here at a time and one of its threads stores them with TMA.
  static constexpr int OFF_STG = OFF_KV + NS * STAGE_BYTES;
  // Row statistics (running max m in log2 units, sum l) of each tile's last unit, two buffers
  // per tile (by the parity of the tile's epilogue count).
  static constexpr int OFF_STATS = OFF_STG + CHUNK;
  static constexpr int STATS_BYTES = 2 * 2 * 128 * 8;
  static constexpr int OFF_BAR = OFF_STATS + STATS_BYTES;
  // q_full, q_empty, kv_full[NS], kv_empty[NS], s_full[2], p_full[2], o_ready[2], o_free[2], drain,
  // stats_ready[2 tiles][2 buffers], stg_ready, stg_free, p_half[2]
  static constexpr int N_BARS = 2 + 2 * NS + 8 + 1 + 4 + 2 + 2;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM_SLOT + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 512;
  __host__ __device__ static constexpr uint32_t s_col(int x) { return (uint32_t)(128 * x); }
  __host__ __device__ static constexpr uint32_t o_col(int x) { return (uint32_t)(256 + D * x); }
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Number of 128-key tiles query tile [qr0, qr0 + 128) needs (0 when the tile is past Lq).
__device__ __forceinline__ int prefill_kv_tiles(const Prefill2Params& p, int qr0) {
  if (qr0 >= p.Lq) return 0;
  int n = (p.Lk + 127) / 128;
  if (p.causal) {
    const int last = min(qr0 + 127, p.Lq - 1);
    n = min(n, (last + (p.Lk - p.Lq)) / 128 + 1);
  }
  return n;
}

struct UnitCoords {
  int b, h, q0;
};

// First query row and query head of tile x (0 = A, 1 = B) of a unit. Sibling pairs (dense mode,
// even group size): heads h and h + 1 of one kv head at the same rows, so both tiles see the same
// key tiles and finish together. Adjacent pairs: rows q0.. and q0 + 128.. of head h (under a
// causal mask tile B has one key tile more, which it processes alone).
__device__ __forceinline__ int tile_row0(const Prefill2Params& p, const UnitCoords& uc, int x) {
  return uc.q0 + (p.sib ? 0 : 128 * x);
}
__device__ __forceinline__ int tile_head(const Prefill2Params& p, const UnitCoords& uc, int x) {
  return uc.h + (p.sib ? x : 0);
}

// The key blocks one query tile processes, in increasing order: 0 .. n-1 in dense mode, the
// caller's list in block-sparse mode.
struct TileList {
  const int32_t* idx;  // nullptr: dense
  int n;
  __device__ __forceinline__ int block(int t) const { return idx ? __ldg(idx + t) : t; }
};

// Tile x (0: rows q0.., 1: rows q0 + 128..) of unit uc. In block-sparse mode the list is read
// up to its first entry that is out of range or not above its predecessor (the kernel then
// records kDevErrBadIndex when `report`) and stops before the first block that lies wholly
// above the causal diagonal of the tile: every later entry would be masked out too.
template <bool SPARSE>
__device__ __forceinline__ TileList prefill_tile_list(const Prefill2Params& p, const UnitCoords& uc, int x,
                                                      bool report) {
  const int qr0 = tile_row0(p, uc, x);
  const int n_dense = prefill_kv_tiles(p, qr0);
  if constexpr (!SPARSE) {
    return TileList{nullptr, n_dense};
  } else {
    if (n_dense == 0) return TileList{nullptr, 0};
    const long long slot = ((long long)uc.b * p.Hq + tile_head(p, uc, x)) * p.n_qblocks + qr0 / 128;
    const int32_t* lst = p.blk_idx + slot * p.max_blk;
    int cnt = __ldg(p.blk_cnt + slot);
    bool bad = cnt < 0 || cnt > p.max_blk;
    if (bad) cnt = 0;
    int n = 0, prev = -1;
    for (int t = 0; t < cnt; ++t) {
      const int kb = __ldg(lst + t);
      if (kb <= prev || kb >= p.n_kblocks) {
        bad = true;
        break;
      }
      if (kb >= n_dense) break;
      prev = kb;
      ++n;
    }
    if (bad && report) raise_bad_index();
    return TileList{lst, n};
  }
}

// Walks the union of the two tiles' block lists in increasing order. Every role of the CTA (TMA
// producer, MMA issuer, softmax warpgroups) derives the same sequence from the same lists.
struct UnionWalk {
  TileList a, b;
  int ia, ib;
  __device__ __forceinline__ UnionWalk(const TileList& la, const TileList& lb) : a(la), b(lb), ia(0), ib(0) {}
  // Next block of the union and which tiles list it; false once both lists are exhausted.
  __device__ __forceinline__ bool next(int& kb, bool& in_a, bool& in_b) {
    const int ka = ia < a.n ? a.block(ia) : 0x7fffffff;
    const int kc = ib < b.n ? b.block(ib) : 0x7fffffff;
    if (ka == 0x7fffffff && kc == 0x7fffffff) return false;
    kb = min(ka, kc);
    in_a = ka == kb;
    in_b = kc == kb;
    ia += in_a ? 1 : 0;
    ib += in_b ? 1 : 0;
    return true;
  }
};

template <bool SPARSE>
__device__ __forceinline__ int union_size(const TileList& la, const TileList& lb) {
  if constexpr (!SPARSE) {
    return max(la.n, lb.n);
  } else {
    UnionWalk w(la, lb);
    int n = 0, kb;
    bool x0, x1;
    while (w.next(kb, x0, x1)) ++n;
    return n;
  }
}

// Unit order. Batches are taken in groups of group_b whose K/V together fits in L2 with room to
// spare; within a group the units are sorted by cost (heaviest level first: under a causal mask
// the cost of a unit grows with its rows' position), then by batch, then by head (pair), so that
// the query heads of a kv head are adjacent and share their K/V tiles in L2. (Taking the
// heaviest pairs of all batches first would keep every batch's K/V live at once and, for a
// 16-batch 2K prefill, doubled the DRAM reads.)
__device__ __forceinline__ UnitCoords prefill_unit(const Prefill2Params& p, int u) {
  // a level is one 128-row query tile (sibling pairs) or one pair of adjacent tiles, heaviest
  // first; a level holds one unit per (batch, head pair) or (batch, head)
  const int n_lvl = p.sib ? p.n_qblocks : p.n_pairs;
  const int hpl = p.sib ? p.Hq / 2 : p.Hq;
  const int per_batch = n_lvl * hpl;
  const int per_group = p.group_b * per_batch;
  const int g = u / per_group;
  const int b0 = g * p.group_b;
  const int gb = min(p.group_b, p.B - b0);
  const int w = u - g * per_group;
  const int lvl = w / (gb * hpl);
  const int rem = w - lvl * gb * hpl;
  UnitCoords c;
  c.b = b0 + rem / hpl;
  c.h = (rem % hpl) * (p.sib ? 2 : 1);
  c.q0 = (n_lvl - 1 - lvl) * (p.sib ? 128 : 256);
  return c;
}

// The k-th unit of CTA `cta` among `grid` persistent CTAs: units are dealt in rounds of `grid`,
// in CTA order on even rounds and in reverse order on odd rounds. On the cost-sorted sequence
// this evens out the per-CTA totals (plain round-robin gives CTA 0 the heaviest unit of every
// round: 12 % longer critical path on an 8K causal prefill).
__device__ __forceinline__ int prefill_unit_index(int k, int cta, int grid) {
  return k * grid + ((k & 1) ? grid - 1 - cta : cta);
}

template <int D, typename E, bool SPARSE>
__global__ void __launch_bounds__(Prefill2Cfg<D>::THREADS, 1)
    prefill2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const Prefill2Params p) {
  using C = Prefill2Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar_q_full = base + C::OFF_BAR;
  const uint32_t bar_q_empty = bar_q_full + 8;
  const uint32_t bar_kv_full = bar_q_empty + 8;
  const uint32_t bar_kv_empty = bar_kv_full + 8 * C::NS;
  const uint32_t bar_s_full = bar_kv_empty + 8 * C::NS;  // [2]
  const uint32_t bar_p_full = bar_s_full + 16;           // [2]
  const uint32_t bar_o_ready = bar_p_full + 16;          // [2]
  const uint32_t bar_o_free = bar_o_ready + 16;          // [2]
  const uint32_t bar_drain = bar_o_free + 16;
  // one barrier per statistics buffer: a tile whose units have a single key tile can hand over
  // two units' statistics before the epilogue waits for the first, and a parity wait on a single
  // barrier could not tell those two phases apart
  const uint32_t bar_stats_ready = bar_drain + 8;  // [tile * 2 + buffer]
  const uint32_t bar_stg_ready = bar_stats_ready + 32;
  const uint32_t bar_stg_free = bar_stg_ready + 8;
  // P of a key tile is handed over in two halves (keys 0-63, then 64-127): the first four P.V
  // products run while the softmax still computes the second half
  const uint32_t bar_p_half = bar_stg_free + 8;  // [2]
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
      mbar_init(bar_p_full + 8 * x, 128);
      mbar_init(bar_p_half + 8 * x, 128);
      mbar_init(bar_o_ready + 8 * x, 1);
      mbar_init(bar_o_free + 8 * x, 128);
    }
    mbar_init(bar_drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar_stats_ready + 8 * i, 128);
    mbar_init(bar_stg_ready, 128);
    mbar_init(bar_stg_free, 1);
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const int wg = warp >> 2;
  // each role starts with its register reallocation, so that the compiler allocates the role's
  // code within that role's count
  if (wg == 3) {
    regs_decrease<80>();
    if (warp == 12) {
      // ------------------------------- TMA producer -------------------------------
      if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      bool ok = true;
      int kv_t = 0, qc = 0;
      // stage kv_t % NS receives K and V of one key tile under a single full barrier
      auto load_kv = [&](int tile, int zkv) {
        const int s = kv_t % C::NS;
        if (kv_t >= C::NS) ok = mbar_wait_inl(bar_kv_empty + 8 * s, ((kv_t / C::NS) & 1) ^ 1, 61);
        if (!ok) return;
        const uint32_t full = bar_kv_full + 8 * s;
        const uint32_t dst = base + C::OFF_KV + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(full, C::STAGE_BYTES);
#pragma unroll
        for (int c = 0; c < C::DC; ++c) tma_load_3d(dst + c * C::CHUNK, &tm_k, full, 64 * c, tile * C::BN, zkv);
#pragma unroll
        for (int c = 0; c < C::DC; ++c)
          tma_load_3d(dst + C::KV_BYTES + c * C::CHUNK, &tm_v, full, 64 * c, tile * C::BN, zkv);
        ++kv_t;
      };
      if constexpr (SPARSE) {
        for (int k = 0, u = blockIdx.x; u < p.n_units && ok; ++k, u = prefill_unit_index(k, blockIdx.x, gridDim.x)) {
          const UnitCoords uc = prefill_unit(p, u);
          const TileList la = prefill_tile_list<SPARSE>(p, uc, 0, true);
          const TileList lb = prefill_tile_list<SPARSE>(p, uc, 1, true);
          if (la.n == 0 && lb.n == 0) continue;  // nothing to load: the softmax writes the empty rows
          if (qc > 0) ok = mbar_wait_inl(bar_q_empty, (qc - 1) & 1, 62);
          if (!ok) break;
          const int zkv = uc.b * p.Hkv + uc.h / p.G;
          mbar_arrive_expect_tx(bar_q_full, ((la.n > 0 ? 1 : 0) + (lb.n > 0 ? 1 : 0)) * C::Q_BYTES);
          for (int x = 0; x < 2; ++x) {
            if ((x == 0 ? la.n : lb.n) == 0) continue;
            const int zq = uc.b * p.Hq + tile_head(p, uc, x);
  #pragma unroll
            for (int c = 0; c < C::DC; ++c)
              tma_load_3d(base + C::OFF_Q + x * C::Q_BYTES + c * C::CHUNK, &tm_q, bar_q_full, 64 * c, tile_row0(p, uc, x), zq);
          }
          ++qc;
          UnionWalk walk(la, lb);
          int kb;
          bool in_a, in_b;
          while (ok && walk.next(kb, in_a, in_b)) load_kv(kb, zkv);
        }
      } else {
        for (int k = 0, u = blockIdx.x; u < p.n_units && ok; ++k, u = prefill_unit_index(k, blockIdx.x, gridDim.x)) {
          const UnitCoords uc = prefill_unit(p, u);
          const int nA = prefill_kv_tiles(p, tile_row0(p, uc, 0)), nB = prefill_kv_tiles(p, tile_row0(p, uc, 1));
          const int n = max(nA, nB);
          if (qc > 0) ok = mbar_wait_inl(bar_q_empty, (qc - 1) & 1, 62);
          if (!ok) break;
          const int zkv = uc.b * p.Hkv + uc.h / p.G;
          mbar_arrive_expect_tx(bar_q_full, (nB > 0 ? 2 : 1) * C::Q_BYTES);
          for (int x = 0; x < (nB > 0 ? 2 : 1); ++x) {
            const int zq = uc.b * p.Hq + tile_head(p, uc, x);
  #pragma unroll
            for (int c = 0; c < C::DC; ++c)
              tma_load_3d(base + C::OFF_Q + x * C::Q_BYTES + c * C::CHUNK, &tm_q, bar_q_full, 64 * c, tile_row0(p, uc, x), zq);
          }
          ++qc;
          for (int j = 0; j < n && ok; ++j) load_kv(j, zkv);
        }
      }
      if (!ok) {
        if (qc > 0) mbar_wait_drain(bar_q_full, (qc - 1) & 1);
        for (int u = max(0, kv_t - C::NS); u < kv_t; ++u) mbar_wait_drain(bar_kv_full + 8 * (u % C::NS), (u / C::NS) & 1);
      }
    }
    } else if (warp == 13) {
    // ------------------------------- MMA issuer -------------------------------
    // The whole warp runs the issuer's control flow and its waits; the lane elected here issues
    // every product and commit. (Run inside a one-lane branch, the same loop issued M128 products
    // more slowly than the tensor core retires them; with warp-uniform control flow the issue cost
    // falls below the math time of a product.)
    {
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_s = make_idesc(C::BM, C::BN, false, false, E::kFmt);
      constexpr uint32_t idesc_o = make_idesc(C::BM, D, false, true, E::kFmt);
      bool ok = true, issued = false;
      int kv_t = 0, qc = 0;
      int p_cnt[2] = {0, 0}, units_done[2] = {0, 0};
      // bounded wait by every lane; the outcome is made warp-uniform
      auto wait_u = [&](uint32_t bar, uint32_t parity, uint32_t site) {
        ok = __all_sync(0xffffffffu, mbar_wait_inl(bar, parity, site));
        return ok;
      };
      auto commit = [&](uint32_t bar) {
        if (leader) mma_commit(bar);
        __syncwarp();
      };
      auto wait_stage = [&](int idx, uint32_t site) {
        if (wait_u(bar_kv_full + 8 * (idx % C::NS), (idx / C::NS) & 1, site)) tc_fence_after();
      };
      auto issue_s = [&](int x, int sidx) {
        const uint32_t kb = base + C::OFF_KV + (sidx % C::NS) * C::STAGE_BYTES;
        const uint32_t qb = base + C::OFF_Q + x * C::Q_BYTES;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = make_sdesc(qb + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = make_sdesc(kb + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024, kSwizzle128B);
            mma_ss(tmem + C::s_col(x), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_s_full + 8 * x);
        }
        __syncwarp();
        issued = true;
      };
      // O_x (+)= P_x V of stage si over keys [64 half, 64 half + 64); `first`: the first block of
      // this tile in the unit (its first product overwrites O)
      auto issue_pv = [&](int x, int si, bool first, int half) {
        const uint32_t vb = base + C::OFF_KV + (si % C::NS) * C::STAGE_BYTES + C::KV_BYTES;
        if (leader) {
#pragma unroll
          for (int kk = half * (C::BN / 32); kk < (half + 1) * (C::BN / 32); ++kk) {
            const uint64_t bd = make_sdesc(vb + kk * 2048, C::CHUNK, 1024, kSwizzle128B);
            // A = P_x in TMEM: keys [16kk, 16kk + 16) are columns [8kk, 8kk + 8) of S_x
            mma_ts(tmem + C::o_col(x), tmem + C::s_col(x) + 8 * kk, bd, idesc_o, (!first || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      // Per key tile j the only wait between the last S product of tile j and the first P.V
      // product of tile j+1 is the one on P: the stage of tile j is released right after its
      // last P.V product (one commit, while the tensor core still has S work queued), and the
      // stage of tile j+1 is awaited before the first S of tile j+1.
      if constexpr (SPARSE) {
        for (int k = 0, u = blockIdx.x; u < p.n_units && ok; ++k, u = prefill_unit_index(k, blockIdx.x, gridDim.x)) {
          const UnitCoords uc = prefill_unit(p, u);
          const TileList lx[2] = {prefill_tile_list<SPARSE>(p, uc, 0, false), prefill_tile_list<SPARSE>(p, uc, 1, false)};
          if (lx[0].n == 0 && lx[1].n == 0) continue;
          const int n = union_size<SPARSE>(lx[0], lx[1]);  // key blocks loaded for this unit
          if (!wait_u(bar_q_full, qc & 1, 63)) break;
          ++qc;
          tc_fence_after();
          UnionWalk walk(lx[0], lx[1]);
          int kb;
          bool in[2];
          walk.next(kb, in[0], in[1]);
          wait_stage(kv_t, 64);  // K, V of the first block
          if (!ok) break;
          for (int x = 0; x < 2; ++x)
            if (in[x]) issue_s(x, kv_t);
          if (n == 1) commit(bar_q_empty);  // the last S of this unit has been issued
          int jx[2] = {0, 0};               // blocks of each tile already multiplied by V
          for (int j = 0; j < n && ok; ++j) {
            const int si = kv_t + j;  // stage of union block j
            bool in_next[2] = {false, false};
            const bool has_next = j + 1 < n && walk.next(kb, in_next[0], in_next[1]);
            const int x_last = in[1] ? 1 : 0;  // last tile whose P.V reads this V
            bool next_ready = false;
            for (int x = 0; x < 2 && ok; ++x) {
              if (in[x]) {
                // previous epilogue read O_x
                if (jx[x] == 0 && units_done[x] > 0 && !wait_u(bar_o_free + 8 * x, (units_done[x] - 1) & 1, 66)) break;
                if (!wait_u(bar_p_half + 8 * x, p_cnt[x] & 1, 74)) break;
                tc_fence_after();
                issue_pv(x, si, jx[x] == 0, 0);
                if (!wait_u(bar_p_full + 8 * x, p_cnt[x] & 1, 67)) break;
                ++p_cnt[x];
                tc_fence_after();
                issue_pv(x, si, false, 1);
                // K was last read by the S products of this block (issued earlier), V by this one
                if (x == x_last) commit(bar_kv_empty + 8 * (si % C::NS));
              }
              if (has_next && in_next[x]) {
                if (!next_ready) {
                  wait_stage(si + 1, 68);  // K, V of the next union block
                  if (!ok) break;
                  next_ready = true;
                }
                issue_s(x, si + 1);
              }
              if (in[x]) {
                if (jx[x] == lx[x].n - 1) {
                  commit(bar_o_ready + 8 * x);
                  ++units_done[x];
                }
                ++jx[x];
              }
            }
            if (!ok) break;
            // Q may be reloaded once the last S of this unit (issued in step n-2) is done
            if (j == n - 2) commit(bar_q_empty);
            in[0] = in_next[0];
            in[1] = in_next[1];
          }
          if (!ok) break;
          kv_t += n;
        }
      } else {
        for (int k = 0, u = blockIdx.x; u < p.n_units && ok; ++k, u = prefill_unit_index(k, blockIdx.x, gridDim.x)) {
          const UnitCoords uc = prefill_unit(p, u);
          int nX[2];
          nX[0] = prefill_kv_tiles(p, tile_row0(p, uc, 0));
          nX[1] = prefill_kv_tiles(p, tile_row0(p, uc, 1));
          const int n = max(nX[0], nX[1]);
          if (!wait_u(bar_q_full, qc & 1, 63)) break;
          ++qc;
          tc_fence_after();
          wait_stage(kv_t, 64);  // K_0, V_0
          if (!ok) break;
          for (int x = 0; x < 2; ++x)
            if (nX[x] > 0) issue_s(x, kv_t);
          if (n == 1) commit(bar_q_empty);  // the last S of this unit has been issued
          for (int j = 0; j < n && ok; ++j) {
            const int si = kv_t + j;                // stage of tile j
            const int x_last = (j < nX[1]) ? 1 : 0;  // last tile whose P.V reads V_j
            bool next_ready = false;
            for (int x = 0; x < 2 && ok; ++x) {
              if (j >= nX[x]) continue;
              // previous epilogue read O_x
              if (j == 0 && units_done[x] > 0 && !wait_u(bar_o_free + 8 * x, (units_done[x] - 1) & 1, 66)) break;
              if (!wait_u(bar_p_half + 8 * x, p_cnt[x] & 1, 74)) break;
              tc_fence_after();
              issue_pv(x, si, j == 0, 0);
              if (!wait_u(bar_p_full + 8 * x, p_cnt[x] & 1, 67)) break;
              ++p_cnt[x];
              tc_fence_after();
              issue_pv(x, si, false, 1);
              // K_j was last read by S of tile j (issued earlier), V_j by this product
              if (x == x_last) commit(bar_kv_empty + 8 * (si % C::NS));
              if (j + 1 < nX[x]) {
                if (!next_ready) {
                  wait_stage(si + 1, 68);  // K_{j+1}, V_{j+1}
                  if (!ok) break;
                  next_ready = true;
                }
                issue_s(x, si + 1);
              }
              if (j == nX[x] - 1) {
                commit(bar_o_ready + 8 * x);
                ++units_done[x];
              }
            }
            if (!ok) break;
            // Q may be reloaded once the last S of this unit (issued in iteration n-2) is done
            if (j == n - 2) commit(bar_q_empty);
          }
          if (!ok) break;
          kv_t += n;
        }
      }
      if (!ok && issued) {
        commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
    }
  } else if (wg == 2) {
    regs_decrease<64>();
    // ------------------------ epilogue warpgroup (warps 8-11) ------------------------
    // For each tile with an output, in the order (unit, tile A, tile B): wait for its last P.V and
    // its row statistics, read O out of TMEM 32 columns at a time (then release O for the next
    // unit), write O / l as 16-bit rows into the staging buffer and store each 64-column chunk
    // with TMA; write LSE.
    const int r = threadIdx.x & 127;  // row of the tile == TMEM lane of this thread
    const uint32_t tw = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t stg = base + C::OFF_STG;
    const float2* stats = reinterpret_cast<const float2*>(smem + C::OFF_STATS);
    int ecnt[2] = {0, 0};  // outputs written per tile
    int stg_uses = 0;      // chunks stored through the staging buffer
    bool ok = true;
    for (int k = 0, u = blockIdx.x; u < p.n_units && ok; ++k, u = prefill_unit_index(k, blockIdx.x, gridDim.x)) {
      const UnitCoords uc = prefill_unit(p, u);
      for (int x = 0; x < 2 && ok; ++x) {
        const int qx0 = tile_row0(p, uc, x);
        if (qx0 >= p.Lq) continue;
        if (SPARSE && prefill_tile_list<SPARSE>(p, uc, x, false).n == 0) continue;  // written by the softmax
        const int par = ecnt[x] & 1;
        ok = mbar_wait_inl(bar_o_ready + 8 * x, par, 70);
        if (ok) ok = mbar_wait_inl(bar_stats_ready + 8 * (2 * x + par), (ecnt[x] >> 1) & 1, 73);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++ecnt[x];
        tc_fence_after();
        const float2 ml = stats[(x * 2 + par) * 128 + r];  // (m in log2 units, l)
        float inv_l = 1.f / ml.y;
        if constexpr (SPARSE) inv_l = ml.y > 0.f ? inv_l : 0.f;  // l = 0: the row saw no key
        const size_t bh = (size_t)uc.b * p.Hq + tile_head(p, uc, x);
        const uint32_t o_col = C::o_col(x);
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          // columns 32*c4 .. +31: 16-byte units 4*(c4 % 2) .. +3 of the 64-column chunk c4 / 2
          if ((c4 & 1) == 0 && stg_uses > 0) {
            ok = mbar_wait_inl(bar_stg_free, (stg_uses - 1) & 1, 71);  // the previous chunk has been read
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          float o[32];
          tmem_ld32(tw + o_col + 32 * c4, o);
          tmem_wait_ld();
          if (c4 == D / 32 - 1) {
            // O has been read out of TMEM: the next unit's first P.V may overwrite it
            tc_fence_before();
            mbar_arrive(bar_o_free + 8 * x);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(stg + swz128_offset((uint32_t)r, (uint32_t)(4 * (c4 & 1) + q)),
                         E::pack2(o[8 * q] * inv_l, o[8 * q + 1] * inv_l), E::pack2(o[8 * q + 2] * inv_l, o[8 * q + 3] * inv_l),
                         E::pack2(o[8 * q + 4] * inv_l, o[8 * q + 5] * inv_l), E::pack2(o[8 * q + 6] * inv_l, o[8 * q + 7] * inv_l));
          if (c4 & 1) {
            fence_proxy_async_smem();  // the staging writes, visible to the TMA engine
            mbar_arrive(bar_stg_ready);
            if (r == 0) {
              // rows past Lq fall outside the tensor map and are not written
              if (mbar_wait_inl(bar_stg_ready, stg_uses & 1, 72)) {
                tma_store_3d(&tm_o, stg, 32 * (c4 - 1), qx0, (int)bh);
                bulk_commit_group();
                bulk_wait_read_all();
              }
              mbar_arrive(bar_stg_free);
            }
            ++stg_uses;
          }
        }
        if (!ok) break;
        const int row = qx0 + r;
        if (row < p.Lq && p.lse != nullptr) {
          float lse_row = (ml.x + log2f(ml.y)) * kLn2;
          if constexpr (SPARSE) lse_row = ml.y > 0.f ? lse_row : -INFINITY;
          p.lse[bh * p.Lq + row] = lse_row;
        }
      }
    }
    if (r == 0) bulk_wait_all();  // this thread's output stores have completed
  } else {
    regs_increase<184>();
    // --------------------------- softmax warpgroups (warps 0-3: A, 4-7: B) ---------------------------
    const int x = warp >> 2;
    const int r = threadIdx.x & 127;  // row of the tile == TMEM lane
    const uint32_t tw = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = C::s_col(x), o_col = C::o_col(x);
    const float c2 = p.scale_log2;
    const int off = p.Lk - p.Lq;
    int s_cnt = 0, e_cnt = 0;  // S tiles consumed; outputs handed to the epilogue warpgroup
    float2* stats = reinterpret_cast<float2*>(smem + C::OFF_STATS);
    bool ok = true;
    for (int k = 0, u = blockIdx.x; u < p.n_units && ok; ++k, u = prefill_unit_index(k, blockIdx.x, gridDim.x)) {
      const UnitCoords uc = prefill_unit(p, u);
      const int qx0 = tile_row0(p, uc, x);
      if (qx0 >= p.Lq) continue;  // tile past the last query row
      const TileList lst = prefill_tile_list<SPARSE>(p, uc, x, false);
      const int nt = lst.n;
      const int row = qx0 + r;
      if (SPARSE && nt == 0) {
        // no listed block: these rows see no key (O = 0, LSE = -inf); nothing was loaded for them
        if (row < p.Lq) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + ((size_t)(uc.b * p.Hq + tile_head(p, uc, x)) * p.Lq + row) * D);
#pragma unroll
          for (int q = 0; q < D / 8; ++q) dst[q] = make_uint4(0u, 0u, 0u, 0u);
          if (p.lse != nullptr) p.lse[(size_t)(uc.b * p.Hq + tile_head(p, uc, x)) * p.Lq + row] = -INFINITY;
        }
        continue;
      }
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < nt; ++j) {
        ok = mbar_wait_inl(bar_s_full + 8 * x, s_cnt & 1, 69);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        float s[4][32];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tw + s_col + 32 * c4, s[c4]);
        tmem_wait_ld();
        int kv0 = j * C::BN;
        if constexpr (SPARSE) kv0 = lst.block(j) * C::BN;
        if (kv0 + C::BN > p.Lk || (p.causal && kv0 + C::BN - 1 > qx0 + off)) {
          int lim = p.Lk - 1;
          if (p.causal) lim = min(lim, row + off);
          const int rem = lim - kv0;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * c4 + e > rem) s[c4][e] = -INFINITY;
        }
        // row max: two independent chains of three-input maxima
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            mx0 = fmax3(mx0, s[c4][e], s[c4][e + 1]);
            mx1 = fmax3(mx1, s[c4][e + 2], s[c4][e + 3]);
          }
        const float mx = fmaxf(mx0, mx1);
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
        // a warp that rescales O hands its first half of P over only after the rescale below (the
        // half barrier waits for all four warps, so no P.V of tile j runs before it)
        const bool resc = __any_sync(0xffffffffu, rescale);
        // p = 2^(s * c2 - m_ref) on key pairs: packed fma, two ex2, packed sum, bf16x2 pack
        const uint64_t c2x2 = f2_pack(c2, c2), nm2 = f2_pack(-m_ref, -m_ref);
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {  // 32 keys -> 16 packed columns at a time
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t xv = ffma2(f2_pack(s[q4][2 * e], s[q4][2 * e + 1]), c2x2, nm2);
            float p0, p1;
            if (kExp2EmulateMask<D> & (1u << e)) {
              // this pair on the FMA pipe: the MUFU unit is the softmax's busiest resource
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
          // P overwrites the S columns it came from: keys 32*q4 .. 32*q4 + 31
          tmem_st16u(tw + s_col + 16 * q4, pk);
          if (q4 == 1 && !resc) {  // keys 0-63 are in place: the first P.V products may start
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p_half + 8 * x);
          }
        }
        float a0, a1, b0, b1;
        f2_unpack(acc0, a0, a1);
        f2_unpack(acc1, b0, b1);
        const float sum = (a0 + a1) + (b0 + b1);
        l += sum;
        // s_full of tile j also covers P.V of tile j-1, so O is stable here
        if (resc) {
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
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
        if (resc) mbar_arrive(bar_p_half + 8 * x);
        mbar_arrive(bar_p_full + 8 * x);
      }
      if (!ok) break;
      // hand the row statistics to the epilogue warpgroup (two buffers: the one written here is
      // read before the next but one unit of this tile can end, since that unit's first P.V waits
      // for the epilogue to release O) and go on with the next unit
      stats[(x * 2 + (e_cnt & 1)) * 128 + r] = make_float2(m_used, l);
      mbar_arrive(bar_stats_ready + 8 * (2 * x + (e_cnt & 1)));
      ++e_cnt;
    }
  }

  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
