// attn_api.cu -- the C ABI of libattn_b200.so (declared in include/attn.h and, for the
// diagnostics, include/attn_diag.h).
//
// Host side only: argument checks, TMA tensor-map encoding (driver entry point looked up once),
// split selection and kernel launches. The kernels live in the .cuh files included below so the
// whole library is one translation unit (one device-side error word, no device linking).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/attn.h"
#include "../../include/attn_diag.h"
#include "combine.cuh"
#include "decode.cuh"
#include "prefill2.cuh"
#include "prefill_pair.cuh"

namespace {

using attn::DecodeParams;

constexpr int kAbiVersion = 10300;  // 1.3.0: attn_decode_default_splits takes the KV layout


typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 16-bit-float tensor map over a row-major [n2, n1, n0] array (n0 contiguous), 128-byte swizzle,
// zero fill out of bounds. box = {b0, b1, 1}. rank 2 when n2 == 0.
template <typename E>
bool encode16(CUtensorMap* map, const void* ptr, uint64_t n0, uint64_t n1, uint64_t n2, uint32_t b0, uint32_t b1,
              uint64_t row_stride = 0) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  const uint64_t rs = row_stride ? row_stride : n0;  // elements between consecutive rows
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {rs * 2, rs * n1 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const cuuint32_t rank = n2 == 0 ? 2 : 3;
  CUresult r = enc(map, E::kFmt == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int current_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Set the dynamic shared-memory limit of a kernel (cheap; done on every launch so that every
// device the caller uses is covered).
template <typename K>
bool allow_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// How many clusters of a kernel can be resident at once on the current device (queried once per
// device and kernel; `fallback` when the query fails).
template <typename K>
int resident_clusters(K kernel, cudaLaunchConfig_t cfg, int fallback) {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return std::max(1, fallback);
  if (cache[dev] > 0) return cache[dev];
  cfg.gridDim = dim3(2u * (unsigned)std::max(1, fallback));
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return std::max(1, fallback);
  }
  cache[dev] = n;
  return n;
}

attn_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status check_common(const void* q, const void* k, const void* v, const void* o, const float* lse, int B, int Hq,
                         int Hkv, int Lq, int Lk, int d, int dv, float scale, int causal) {
  if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || d < 1 || dv < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * Hq > 0x7fffffffLL || (long long)B * Hq * Lq > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return ATTN_ERR_MISALIGNED;
  if (lse && !aligned(lse, 4)) return ATTN_ERR_MISALIGNED;
  return ATTN_OK;
}

// ---------------------------------------------------------------------------------------------
// decode: split selection and workspace layout
// ---------------------------------------------------------------------------------------------
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t workspace_bytes(long long rows, int dv, int splits) {
  return align256((size_t)splits * rows * dv * 4) + align256((size_t)splits * rows * 4);
}

bool tc_supported(const void* k, const void* v, int Hq, int Hkv, int Lq, int d, int dv, int ldv) {
  const int R = (Hq / Hkv) * Lq;
  return v == k && ldv == d && d % 64 == 0 && d <= 576 && dv % 128 == 0 && dv <= 512 && dv <= d && R <= 32;
}

// queries-on-M kernel: latent KV as above, or a dense separate V with dv == d (GQA decode)
bool tn_supported(const void* k, const void* v, int Hq, int Hkv, int Lq, int d, int dv, int ldv) {
  if (tc_supported(k, v, Hq, Hkv, Lq, d, dv, ldv)) return true;
  const int R = (Hq / Hkv) * Lq;
  return v != k && dv == d && (d == 128 || d == 256) && ldv % 8 == 0 && R <= 32;
}

bool cc_supported(int Hq, int Hkv, int Lq, int d, int dv, int ldv) {
  const int R = (Hq / Hkv) * Lq;
  return R <= 64 && d <= 576 && dv <= 512 && d % 8 == 0 && dv % 8 == 0 && ldv % 8 == 0 && ldv >= dv;
}

// Keys per split: a multiple of 64.
int split_chunk(int Lk, int splits) {
  int c = (Lk + splits - 1) / splits;
  return (c + 63) / 64 * 64;
}

// Choose the split count of the equal-chunk grid. Model: CTAs run ctas_per_sm per SM in waves; a
// CTA costs its key tiles plus a fixed start-up/drain cost of about kFixedTiles tiles (barrier
// set-up, Q load, ring fill, partial write), and every split adds partial-result traffic. Minimise
//   waves * (tiles per split + kFixedTiles) * (1 + partial bytes / KV bytes).
// (On B200: mla_decode_64k -> 9 splits at one CTA per SM, gqa_decode_32k -> 9 at two CTAs per
// SM, both the measured best: 4 to 28 splits were timed.)
int choose_splits(int B, int Hq, int Hkv, int Lq, int Lk, int dv, int sms, int ctas_per_sm) {
  constexpr double kFixedTiles = 5.0, kTileKeys = 48.0;
  const long long units = (long long)B * Hkv;
  const long long rows = (long long)B * Hq * Lq;
  const double kv_bytes = (double)units * Lk * (double)dv * 2.0;
  const int max_s = std::max(1, std::min(256, Lk / 256));
  int best = 1;
  double best_cost = 1e300;
  for (int s = 1; s <= max_s; ++s) {
    const int chunk = split_chunk(Lk, s);
    const int used = (Lk + chunk - 1) / chunk;  // splits that hold keys
    if (used < s) continue;
    const double slots = (double)sms * ctas_per_sm;
    const double waves = std::ceil((double)(units * s) / slots);
    const double partial = 2.0 * (double)s * rows * (dv + 1) * 4.0 / kv_bytes;
    const double cost = waves * (std::ceil(chunk / kTileKeys) + kFixedTiles) * (1.0 + partial);
    if (cost < best_cost * (1.0 - 1e-9)) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

// CTAs per SM of the dense-V (d = 128) queries-on-M decode kernel: bounded by shared memory
// (228 KB per SM, 1 KB reserved per CTA) and by TMEM (512 columns, 256 per CTA).
using DenseTn128Cfg = attn::DecodeTnCfg<2, 1, 48, 3, true>;
constexpr int kDenseTn128Occupancy = 233472 / (DenseTn128Cfg::SMEM_BYTES + 1024);
static_assert(kDenseTn128Occupancy == 2, "dense-V decode sized for two CTAs per SM");

// Which kernel attn_decode runs for impl == ATTN_DECODE_AUTO.
int auto_impl(const void* k, const void* v, int Hq, int Hkv, int Lq, int d, int dv, int ldv) {
  return tn_supported(k, v, Hq, Hkv, Lq, d, dv, ldv) ? ATTN_DECODE_TCGEN05_N : ATTN_DECODE_CUDA_CORE;
}

// CTAs per SM the split model assumes for a (resolved) kernel choice.
int decode_ctas_per_sm(int impl, bool dense_v, int d) {
  return (impl == ATTN_DECODE_TCGEN05_N && dense_v && d == 128) ? kDenseTn128Occupancy : 1;
}

// How a decode call cuts the keys. Split mode: `splits` equal chunks of every unit (grid
// splits x units). Balanced mode (queries-on-M kernel, num_splits == 0): one CTA per slot of the
// GPU, each taking bal_w consecutive keys of the flattened (unit, key) space, bal_w <= Lk so a
// CTA touches at most two units; `splits` is then the most partials any unit gets.
struct DecodePlan {
  int splits;
  int bal_w;
  long long ctas;
};

DecodePlan balanced_plan(long long units, int Lk, int slots) {
  DecodePlan d{0, 0, 0};
  const long long total = units * Lk;
  long long w = (total + slots - 1) / slots;
  w = (w + 63) / 64 * 64;
  if (w > Lk || w > 0x7fffffffLL) return d;  // a CTA would span more than two units
  int most = 1;
  for (long long u = 0; u < units; ++u) {
    const long long pieces = ((u + 1) * Lk - 1) / w - (u * Lk) / w + 1;
    most = (int)std::max<long long>(most, pieces);
  }
  if (most > 256) return d;
  d.splits = most;
  d.bal_w = (int)w;
  d.ctas = (total + w - 1) / w;
  return d;
}

DecodePlan plan_decode(int impl, bool dense_v, int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, int num_splits) {
  if (num_splits > 0) return DecodePlan{num_splits, 0, 0};
  const int sms = current_sm_count();
  const int occ = decode_ctas_per_sm(impl, dense_v, d);
  if (impl == ATTN_DECODE_TCGEN05_N) {
    const DecodePlan bal = balanced_plan((long long)B * Hkv, Lk, sms * occ);
    if (bal.bal_w > 0) return bal;
  }
  return DecodePlan{choose_splits(B, Hq, Hkv, Lq, Lk, dv, sms, occ), 0, 0};
}

template <int RMAX, int CPT, typename E>
attn_status launch_cc(const DecodeParams& p, int splits, cudaStream_t st) {
  const size_t smem = attn::decode_cc_smem_bytes(p.R, p.d, p.dv, !p.v_is_k);
  auto kern = attn::decode_cc_kernel<RMAX, CPT, E>;
  if (smem > 48 * 1024 && !allow_smem(kern, (int)smem)) return ATTN_ERR_CUDA;
  dim3 grid(splits, p.B * p.Hkv);
  kern<<<grid, attn::kCcThreads, smem, st>>>(p);
  return launch_status();
}

template <int DCH, int NB, int NP, typename E>
attn_status launch_tc(const DecodeParams& p, int splits, cudaStream_t st) {
  using C = attn::DecodeTcCfg<DCH, NB, NP>;
  CUtensorMap tq, tkv;
  if (!encode16<E>(&tq, p.q, (uint64_t)p.d, (uint64_t)p.rows_total, 0, 64, NP)) return ATTN_ERR_CUDA;
  if (!encode16<E>(&tkv, p.k, (uint64_t)p.d, (uint64_t)p.Lk, (uint64_t)p.B * p.Hkv, 64, C::BKV)) return ATTN_ERR_CUDA;
  auto kern = attn::decode_tc_kernel<DCH, NB, NP, E>;
  if (!allow_smem(kern, C::SMEM_BYTES)) return ATTN_ERR_CUDA;
  dim3 grid(splits, p.B * p.Hkv);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tkv, p);
  return launch_status();
}

template <int DCH, int NB, typename E>
attn_status launch_tc_np(const DecodeParams& p, int splits, cudaStream_t st) {
  if (p.R <= 16) return launch_tc<DCH, NB, 16, E>(p, splits, st);
  return launch_tc<DCH, NB, 32, E>(p, splits, st);
}

template <int DCH, typename E>
attn_status launch_tc_nb(const DecodeParams& p, int splits, cudaStream_t st) {
  switch (p.dv / 128) {
    // V^T block nb reads 64-column chunks 2nb and 2nb+1 of the latent tile, so 2*NB <= DCH
    case 1: if constexpr (2 <= DCH) return launch_tc_np<DCH, 1, E>(p, splits, st); else return ATTN_ERR_UNSUPPORTED;
    case 2: if constexpr (4 <= DCH) return launch_tc_np<DCH, 2, E>(p, splits, st); else return ATTN_ERR_UNSUPPORTED;
    case 3: if constexpr (6 <= DCH) return launch_tc_np<DCH, 3, E>(p, splits, st); else return ATTN_ERR_UNSUPPORTED;
    case 4: if constexpr (8 <= DCH) return launch_tc_np<DCH, 4, E>(p, splits, st); else return ATTN_ERR_UNSUPPORTED;
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

#ifndef ATTN_TN_BK
#define ATTN_TN_BK 48
#endif
#ifndef ATTN_TN_NST
#define ATTN_TN_NST 3
#endif
// Key tile and stage count of the queries-on-M decode kernel (chosen by measurement on B200).
constexpr int kTnBK = ATTN_TN_BK, kTnNST = ATTN_TN_NST;

template <int DCH, int NPIECE, int NST, bool SEPV, typename E, int BK = kTnBK>
attn_status launch_tn(const DecodeParams& p, int splits, cudaStream_t st) {
  using C = attn::DecodeTnCfg<DCH, NPIECE, BK, NST, SEPV>;
  CUtensorMap tq, tkv, tv;
  if (!encode16<E>(&tq, p.q, (uint64_t)p.d, (uint64_t)p.rows_total, 0, 64, 32)) return ATTN_ERR_CUDA;
  if (!encode16<E>(&tkv, p.k, (uint64_t)p.d, (uint64_t)p.Lk, (uint64_t)p.B * p.Hkv, 64, BK)) return ATTN_ERR_CUDA;
  if (SEPV) {
    if (!encode16<E>(&tv, p.v, (uint64_t)p.dv, (uint64_t)p.Lk, (uint64_t)p.B * p.Hkv, 64, BK, (uint64_t)p.ldv))
      return ATTN_ERR_CUDA;
  } else {
    tv = tkv;  // unused
  }
  auto kern = attn::decode_tn_kernel<DCH, NPIECE, BK, NST, SEPV, E>;
  if (!allow_smem(kern, C::SMEM_BYTES)) return ATTN_ERR_CUDA;
  dim3 grid(splits, p.B * p.Hkv);
  if (p.bal_w > 0) grid = dim3((unsigned)((p.bal_total + p.bal_w - 1) / p.bal_w), 1);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tkv, tv, p);
  return launch_status();
}

template <int DCH, typename E>
attn_status launch_tn_np(const DecodeParams& p, int splits, cudaStream_t st) {
  if (p.dv <= 256) return launch_tn<DCH, 1, kTnNST, false, E>(p, splits, st);
  return launch_tn<DCH, 2, kTnNST, false, E>(p, splits, st);
}

template <typename E>
attn_status launch_tn_any(const DecodeParams& p, int splits, cudaStream_t st) {
  if (!p.v_is_k) {
    // dense V beside K in each stage; d = 128: a 3-stage ring small enough for two CTAs per SM
    // (each CTA's start-up, drain and per-tile waits hide behind the other's streaming)
    if (p.d == 128) return launch_tn<2, 1, 3, true, E, 48>(p, splits, st);
    if (p.d == 256) return launch_tn<4, 1, 3, true, E>(p, splits, st);
    return ATTN_ERR_UNSUPPORTED;
  }
  switch (p.d / 64) {
    case 2: return launch_tn_np<2, E>(p, splits, st);
    case 3: return launch_tn_np<3, E>(p, splits, st);
    case 4: return launch_tn_np<4, E>(p, splits, st);
    case 5: return launch_tn_np<5, E>(p, splits, st);
    case 6: return launch_tn_np<6, E>(p, splits, st);
    case 7: return launch_tn_np<7, E>(p, splits, st);
    case 8: return launch_tn_np<8, E>(p, splits, st);
    case 9: return launch_tn_np<9, E>(p, splits, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

template <typename E>
attn_status launch_tc_any(const DecodeParams& p, int splits, cudaStream_t st) {
  switch (p.d / 64) {
    case 2: return launch_tc_nb<2, E>(p, splits, st);
    case 3: return launch_tc_nb<3, E>(p, splits, st);
    case 4: return launch_tc_nb<4, E>(p, splits, st);
    case 5: return launch_tc_nb<5, E>(p, splits, st);
    case 6: return launch_tc_nb<6, E>(p, splits, st);
    case 7: return launch_tc_nb<7, E>(p, splits, st);
    case 8: return launch_tc_nb<8, E>(p, splits, st);
    case 9: return launch_tc_nb<9, E>(p, splits, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

template <typename E>
attn_status launch_combine(const float* o_part, const float* lse_part, void* o, float* lse, long long rows, int dv,
                           int splits, cudaStream_t st, int bal_w = 0, int Lk = 0, int R = 1) {
  if (rows <= 0) return ATTN_OK;
  // programmatic dependent launch: the combine's CTAs may be scheduled while the previous kernel
  // on the stream (the decode) drains; the kernel waits for that grid before reading partials
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(attn::kCombineThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, attn::combine_kernel<E>, o_part, lse_part, reinterpret_cast<uint16_t*>(o), lse, rows,
                         dv, splits, bal_w, Lk, R) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return launch_status();
}

// One CTA waits on a barrier that never completes; the bounded wait gives up after limit_ns.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = attn::smem_u32(&bar);
  if (threadIdx.x == 0) {
    attn::mbar_init(b, 1);
    attn::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!attn::mbar_try_wait(b, 0)) (void)attn::mbar_wait_slow(b, 0, 0xEE, limit_ns);
  }
  __syncthreads();
}

// y[i] = 2^x[i] through the FMA-pipe polynomial used by the prefill softmax.
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    float a, b;
    attn::f2_unpack(attn::exp2_poly2(attn::f2_pack(x[i], x[i + 1])), a, b);
    y[i] = a;
    y[i + 1] = b;
  } else if (i < n) {
    float a, b;
    attn::f2_unpack(attn::exp2_poly2(attn::f2_pack(x[i], 0.f)), a, b);
    y[i] = a;
  }
}

}  // namespace

namespace {

// --- typed entry points: dispatch on the element type ---
bool valid_dtype(int dtype) { return dtype == ATTN_DTYPE_BF16 || dtype == ATTN_DTYPE_F16; }

template <typename Fn>
attn_status with_elem(int dtype, Fn&& fn) {
  if (dtype == ATTN_DTYPE_BF16) return fn(attn::ElemBf16{});
  if (dtype == ATTN_DTYPE_F16) return fn(attn::ElemF16{});
  return ATTN_ERR_INVALID_ARG;
}

// Block lists of the sparse mode (all nullptr / 0 in dense mode).
struct SparseBlocks {
  const int32_t* idx;
  const int32_t* cnt;
  int max_blk;
};

template <typename E, bool SPARSE>
attn_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
                     int Lk, int d, float scale, int causal, SparseBlocks sb, void* stream) {
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int n_qtiles = (Lq + 127) / 128;
  CUtensorMap tq, tk, tv, to;
  if (!encode16<E>(&tq, q, (uint64_t)d, (uint64_t)Lq, (uint64_t)B * Hq, 64, 128) ||
      !encode16<E>(&to, o, (uint64_t)d, (uint64_t)Lq, (uint64_t)B * Hq, 64, 128) ||
      !encode16<E>(&tk, k, (uint64_t)d, (uint64_t)Lk, (uint64_t)B * Hkv, 64, 128) ||
      !encode16<E>(&tv, v, (uint64_t)d, (uint64_t)Lk, (uint64_t)B * Hkv, 64, 128))
    return ATTN_ERR_CUDA;
  attn::Prefill2Params p{};
  p.o = reinterpret_cast<uint16_t*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lk = Lk;
  p.G = Hq / Hkv;
  p.n_pairs = (n_qtiles + 1) / 2;
  // dense mode with an even group size: a unit is two sibling query heads of one kv head at the
  // same 128 rows (equal key ranges); otherwise two adjacent row tiles of one head
  p.sib = (!SPARSE && (Hq / Hkv) % 2 == 0) ? 1 : 0;
  const long long units = p.sib ? (long long)n_qtiles * B * (Hq / 2) : (long long)p.n_pairs * B * Hq;
  if (units > 0x7fff0000LL) return ATTN_ERR_UNSUPPORTED;  // room for one more round of unit ids
  p.n_units = (int)units;
  // scheduling groups of batches whose K/V (Hkv * Lk rows of d + dv elements each) stays within
  // 64 MiB, about half of the L2
  const long long kv_per_batch = (long long)Hkv * Lk * (d + d) * 2;
  p.group_b = (int)std::max(1LL, std::min<long long>(B, (64LL << 20) / std::max(1LL, kv_per_batch)));
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.blk_idx = sb.idx;
  p.blk_cnt = sb.cnt;
  p.max_blk = sb.max_blk;
  p.n_qblocks = n_qtiles;
  p.n_kblocks = (Lk + 127) / 128;
#ifndef ATTN_PREFILL_PAIR
#define ATTN_PREFILL_PAIR 0
#endif
  // d = 128, dense key ranges, even GQA groups: the kernel whose products span a pair of SMs
  if (ATTN_PREFILL_PAIR && !SPARSE && d == 128 && (Hq / Hkv) % 2 == 0) {
    CUtensorMap tkh;  // K in boxes of 64 keys: each CTA of a pair loads half of a key tile
    if (!encode16<E>(&tkh, k, (uint64_t)d, (uint64_t)Lk, (uint64_t)B * Hkv, 64, 64)) return ATTN_ERR_CUDA;
    const long long pair_units = (long long)p.n_pairs * B * (Hq / 2);
    if (pair_units > 0x7fff0000LL) return ATTN_ERR_UNSUPPORTED;
    p.n_units = (int)pair_units;
    auto kern = attn::prefill_pair_kernel<E>;
    if (!allow_smem(kern, attn::PairCfg::SMEM_BYTES)) return ATTN_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(attn::PairCfg::THREADS);
    cfg.dynamicSmemBytes = attn::PairCfg::SMEM_BYTES;
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent grid: as many pairs as can be resident at once (SM pairs must share a GPC)
    const int pairs = (int)std::min<long long>(pair_units, resident_clusters(kern, cfg, current_sm_count() / 2));
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    if (cudaLaunchKernelEx(&cfg, kern, tq, tkh, tv, p) != cudaSuccess) return ATTN_ERR_CUDA;
    return launch_status();
  }
  // persistent grid: one CTA per SM (fewer when there are fewer work units)
  const int grid = (int)std::min<long long>(units, current_sm_count());
  if (d == 128) {
    using C = attn::Prefill2Cfg<128>;
    if (!allow_smem(attn::prefill2_kernel<128, E, SPARSE>, C::SMEM_BYTES)) return ATTN_ERR_CUDA;
    attn::prefill2_kernel<128, E, SPARSE><<<grid, C::THREADS, C::SMEM_BYTES, cs>>>(tq, tk, tv, to, p);
  } else {
    using C = attn::Prefill2Cfg<64>;
    if (!allow_smem(attn::prefill2_kernel<64, E, SPARSE>, C::SMEM_BYTES)) return ATTN_ERR_CUDA;
    attn::prefill2_kernel<64, E, SPARSE><<<grid, C::THREADS, C::SMEM_BYTES, cs>>>(tq, tk, tv, to, p);
  }
  return launch_status();
}

// Every argument check of a decode call that does not involve the workspace; on success *impl
// holds the resolved kernel choice (ATTN_DECODE_AUTO replaced).
attn_status check_decode(const void* q, const void* k, const void* v, const void* o, const float* lse, int B, int Hq,
                         int Hkv, int Lq, int Lk, int d, int dv, int ldv, float scale, int causal, int num_splits,
                         int* impl) {
  attn_status st = check_common(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, scale, causal);
  if (st != ATTN_OK) return st;
  if (ldv < dv) return ATTN_ERR_INVALID_ARG;
  if (num_splits < 0 || num_splits > 256) return ATTN_ERR_INVALID_ARG;
  if (*impl < ATTN_DECODE_AUTO || *impl > ATTN_DECODE_TCGEN05_N) return ATTN_ERR_INVALID_ARG;
  if (d % 8 != 0 || dv % 8 != 0 || ldv % 8 != 0) return ATTN_ERR_MISALIGNED;
  if (*impl == ATTN_DECODE_AUTO) *impl = auto_impl(k, v, Hq, Hkv, Lq, d, dv, ldv);
  if (*impl == ATTN_DECODE_TCGEN05_T && !tc_supported(k, v, Hq, Hkv, Lq, d, dv, ldv)) return ATTN_ERR_UNSUPPORTED;
  if (*impl == ATTN_DECODE_TCGEN05_N && !tn_supported(k, v, Hq, Hkv, Lq, d, dv, ldv)) return ATTN_ERR_UNSUPPORTED;
  if (*impl == ATTN_DECODE_CUDA_CORE && !cc_supported(Hq, Hkv, Lq, d, dv, ldv)) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

template <typename E>
attn_status decode_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int Lq, int Lk, int d, int dv, int ldv, float scale, int causal, int num_splits,
                        void* workspace, size_t ws_bytes, int impl, void* stream) {
  attn_status st = check_decode(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, num_splits, &impl);
  if (st != ATTN_OK) return st;
  const bool dense_v = !(v == k && ldv == d);
  const DecodePlan plan = plan_decode(impl, dense_v, B, Hq, Hkv, Lq, Lk, d, dv, num_splits);
  const int splits = plan.splits;
  const long long rows = (long long)B * Hq * Lq;
  const size_t need = workspace_bytes(rows, dv, splits);
  if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return ATTN_ERR_WORKSPACE;

  DecodeParams p{};
  p.q = reinterpret_cast<const uint16_t*>(q);
  p.k = reinterpret_cast<const uint16_t*>(k);
  p.v = reinterpret_cast<const uint16_t*>(v);
  p.o_part = reinterpret_cast<float*>(workspace);
  p.lse_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + align256((size_t)splits * rows * dv * 4));
  p.rows_total = rows;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lk = Lk;
  p.d = d;
  p.dv = dv;
  p.ldv = ldv;
  p.G = Hq / Hkv;
  p.R = p.G * Lq;
  p.causal = causal ? 1 : 0;
  p.chunk = split_chunk(Lk, splits);
  p.v_is_k = (v == k && ldv == d) ? 1 : 0;
  p.bal_w = plan.bal_w;
  p.bal_total = (long long)B * Hkv * Lk;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  if (impl == ATTN_DECODE_TCGEN05_T) {
    st = launch_tc_any<E>(p, splits, cs);
  } else if (impl == ATTN_DECODE_TCGEN05_N) {
    st = launch_tn_any<E>(p, splits, cs);
  } else {
    const int cpt = (dv + attn::kCcThreads - 1) / attn::kCcThreads;
    if (p.R <= 16) st = cpt == 1 ? launch_cc<16, 1, E>(p, splits, cs) : launch_cc<16, 2, E>(p, splits, cs);
    else if (p.R <= 32) st = cpt == 1 ? launch_cc<32, 1, E>(p, splits, cs) : launch_cc<32, 2, E>(p, splits, cs);
    else st = cpt == 1 ? launch_cc<64, 1, E>(p, splits, cs) : launch_cc<64, 2, E>(p, splits, cs);
  }
  if (st != ATTN_OK) return st;
  return launch_combine<E>(p.o_part, p.lse_part, o, lse, rows, dv, splits, cs, p.bal_w, Lk, p.R);
}

}  // namespace

extern "C" {

const char* attn_status_string(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape";
    case ATTN_ERR_MISALIGNED: return "misaligned pointer or stride";
    case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "a bounded wait on the GPU ran out";
  }
  return "unknown status";
}

int attn_abi_version(void) { return kAbiVersion; }

attn_status attn_fwd_typed(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                           int Lq, int Lk, int d, int dv, float scale, int causal, int dtype, void* stream) {
  if (!valid_dtype(dtype)) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_common(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, scale, causal);
  if (st != ATTN_OK) return st;
  if (d != dv || (d != 64 && d != 128)) return ATTN_ERR_UNSUPPORTED;
  return with_elem(dtype, [&](auto e) {
    return fwd_impl<decltype(e), false>(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, causal,
                                        SparseBlocks{nullptr, nullptr, 0}, stream);
  });
}

attn_status attn_fwd_sparse_typed(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                                  int Hkv, int Lq, int Lk, int d, int dv, float scale, int causal,
                                  const int32_t* block_idx, const int32_t* block_cnt, int max_blocks, int dtype,
                                  void* stream) {
  if (!valid_dtype(dtype)) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_common(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, scale, causal);
  if (st != ATTN_OK) return st;
  if (!block_idx || !block_cnt || max_blocks < 1) return ATTN_ERR_INVALID_ARG;
  if (!aligned(block_idx, 4) || !aligned(block_cnt, 4)) return ATTN_ERR_MISALIGNED;
  if (d != dv || (d != 64 && d != 128)) return ATTN_ERR_UNSUPPORTED;
  const long long n_lists = (long long)B * Hq * ((Lq + 127) / 128);
  if (n_lists * max_blocks > (1LL << 40)) return ATTN_ERR_UNSUPPORTED;
  return with_elem(dtype, [&](auto e) {
    return fwd_impl<decltype(e), true>(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, causal,
                                       SparseBlocks{block_idx, block_cnt, max_blocks}, stream);
  });
}

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
                     int Lk, int d, int dv, float scale, int causal, void* stream) {
  return attn_fwd_typed(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, scale, causal, ATTN_DTYPE_BF16, stream);
}

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int dv, int num_splits) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || dv < 1 || num_splits < 0 || num_splits > 256) return 0;
  if (Hq % Hkv != 0) return 0;
  if (num_splits > 0) return workspace_bytes((long long)B * Hq * Lq, dv, num_splits);
  // enough for whatever attn_decode plans for this shape: either kernel family, either occupancy
  int most = 1;
  for (int impl : {ATTN_DECODE_TCGEN05_N, ATTN_DECODE_CUDA_CORE})
    for (bool dense : {false, true})
      for (int dd : {128, 0})
        most = std::max(most, plan_decode(impl, dense, B, Hq, Hkv, Lq, Lk, dd, dv, 0).splits);
  return workspace_bytes((long long)B * Hq * Lq, dv, most);
}

int attn_decode_default_splits(int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, int latent) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || d < 1 || dv < 1 || Hq % Hkv != 0) return 0;
  // the kernel attn_decode picks for this layout (pointers only matter as "v == k or not")
  const void* k = reinterpret_cast<const void*>(uintptr_t(0x100));
  const void* v = latent ? k : reinterpret_cast<const void*>(uintptr_t(0x200));
  const int ldv = latent ? d : dv;
  const int impl = auto_impl(k, v, Hq, Hkv, Lq, d, dv, ldv);
  return plan_decode(impl, !latent, B, Hq, Hkv, Lq, Lk, d, dv, 0).splits;
}

attn_status attn_decode_typed(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                              int Lq, int Lk, int d, int dv, int ldv, float scale, int causal, int num_splits,
                              void* workspace, size_t ws_bytes, int impl, int dtype, void* stream) {
  if (!valid_dtype(dtype)) return ATTN_ERR_INVALID_ARG;
  return with_elem(dtype, [&](auto e) {
    return decode_impl<decltype(e)>(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, num_splits,
                                    workspace, ws_bytes, impl, stream);
  });
}

attn_status attn_decode_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                           int Lq, int Lk, int d, int dv, int ldv, float scale, int causal, int num_splits,
                           void* workspace, size_t ws_bytes, int impl, void* stream) {
  return attn_decode_typed(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, num_splits, workspace,
                           ws_bytes, impl, ATTN_DTYPE_BF16, stream);
}

attn_status attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int Lq, int Lk, int d, int dv, int ldv, float scale, int causal, int num_splits,
                        void* workspace, size_t ws_bytes, void* stream) {
  return attn_decode_ex(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, num_splits, workspace,
                        ws_bytes, ATTN_DECODE_AUTO, stream);
}

// ---------------------------------------------------------------------------------------------
// Allocation-free decode: split partials live in a scratch array compiled into the library.
// ---------------------------------------------------------------------------------------------
}  // extern "C"

namespace {

// The scratch array. In host code its name is only a stand-in for the symbol; kernels must be
// given the device address looked up below.
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Driver entry points used to tell contexts apart (looked up once).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Set-up, done once per device: the device address of the scratch array, looked up with that
// device current. The address belongs to the device's (primary) context; the lookup is tagged
// with the context's unique id and repeated if the context has changed since (a cudaDeviceReset
// destroys the context and its copy of the array, and the next context may place it elsewhere).
struct ScratchAddr {
  void* ptr;
  unsigned long long ctx_id;
};
std::mutex g_scratch_mu;
ScratchAddr g_scratch[kMaxDevices] = {};

attn_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  // no current context yet (first runtime call on this thread): the lookup below creates it
  unsigned long long ctx_id = 0;
  const bool have_ctx = current_context_id(&ctx_id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!have_ctx || g_scratch[dev].ptr == nullptr || g_scratch[dev].ctx_id != ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || p == nullptr) return ATTN_ERR_CUDA;
    if (!current_context_id(&ctx_id)) return ATTN_ERR_CUDA;
    g_scratch[dev] = ScratchAddr{p, ctx_id};
  }
  *out = g_scratch[dev].ptr;
  return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                                int Hkv, int Lq, int Lk, int d, int dv, int ldv, float scale, int causal,
                                int num_splits, void* stream) {
  // the same checks, in the same order, as attn_decode's; only then the scratch size
  int impl = ATTN_DECODE_AUTO;
  attn_status st = check_decode(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, num_splits, &impl);
  if (st != ATTN_OK) return st;
  const DecodePlan plan = plan_decode(impl, !(v == k && ldv == d), B, Hq, Hkv, Lq, Lk, d, dv, num_splits);
  const size_t need = workspace_bytes((long long)B * Hq * Lq, dv, plan.splits);
  if (need > (size_t)ATTN_DECODE_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != ATTN_OK) return st;
  return attn_decode_ex(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, num_splits, scratch,
                        (size_t)ATTN_DECODE_NOALLOC_SCRATCH_BYTES, ATTN_DECODE_AUTO, stream);
}

attn_status attn_combine_typed(const float* o_part, const float* lse_part, void* o, float* lse, int B, int Hq,
                               int Lq, int dv, int num_splits, int dtype, void* stream) {
  if (!valid_dtype(dtype)) return ATTN_ERR_INVALID_ARG;
  if (!o_part || !lse_part || !o) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Lq < 1 || dv < 1 || num_splits < 1 || num_splits > 4096) return ATTN_ERR_INVALID_ARG;
  if (dv % 4 != 0) return ATTN_ERR_MISALIGNED;
  if (!aligned(o_part, 16) || !aligned(lse_part, 4) || !aligned(o, 8) || (lse && !aligned(lse, 4)))
    return ATTN_ERR_MISALIGNED;
  const long long rows = (long long)B * Hq * Lq;
  if (rows > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  return with_elem(dtype, [&](auto e) {
    return launch_combine<decltype(e)>(o_part, lse_part, o, lse, rows, dv, num_splits,
                                       reinterpret_cast<cudaStream_t>(stream));
  });
}

attn_status attn_combine(const float* o_part, const float* lse_part, void* o, float* lse, int B, int Hq, int Lq,
                         int dv, int num_splits, void* stream) {
  return attn_combine_typed(o_part, lse_part, o, lse, B, Hq, Lq, dv, num_splits, ATTN_DTYPE_BF16, stream);
}

attn_status attn_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return ATTN_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)limit_us * 1000ull);
  return launch_status();
}

attn_status attn_selftest_exp2(const float* x, float* y, int n, void* stream) {
  if (!x || !y || n < 1) return ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(y, 4)) return ATTN_ERR_MISALIGNED;
  const int threads = 256, pairs = (n + 1) / 2;
  selftest_exp2_kernel<<<(pairs + threads - 1) / threads, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

}  // extern "C"

namespace {

// ---------------------------------------------------------------------------------------------
// Host-buffer forward: copy-in, compute and copy-out pipelined over pieces of the unit grid.
// ---------------------------------------------------------------------------------------------
constexpr int kHostMaxPieces = 64;

// Per-device streams and events of the host pipeline, created on first use and kept for the
// life of the process (streams and events hold no device memory). One mutex per device
// serialises the host-side enqueue of concurrent calls, which share the events.
struct HostPipe {
  std::mutex mu;
  bool ready = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t e_entry = nullptr, e_done = nullptr;
  cudaEvent_t e_in[kHostMaxPieces] = {}, e_run[kHostMaxPieces] = {};
};
HostPipe g_host_pipe[kMaxDevices];

bool host_pipe_init(HostPipe& hp) {
  if (hp.ready) return true;
  const unsigned ef = cudaEventDisableTiming;
  if (cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaEventCreateWithFlags(&hp.e_entry, ef) != cudaSuccess) return false;
  if (cudaEventCreateWithFlags(&hp.e_done, ef) != cudaSuccess) return false;
  for (int i = 0; i < kHostMaxPieces; ++i)
    if (cudaEventCreateWithFlags(&hp.e_in[i], ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.e_run[i], ef) != cudaSuccess)
      return false;
  hp.ready = true;
  return true;
}

struct HostLayout {
  size_t q, k, v, o, lse, total;  // byte offsets in the device scratch
};

HostLayout host_layout(int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv) {
  HostLayout L{};
  const size_t e = 2;  // 16-bit elements
  L.q = 0;
  L.k = align256(L.q + (size_t)B * Hq * Lq * d * e);
  L.v = align256(L.k + (size_t)B * Hkv * Lk * d * e);
  L.o = align256(L.v + (size_t)B * Hkv * Lk * dv * e);
  L.lse = align256(L.o + (size_t)B * Hq * Lq * dv * e);
  L.total = align256(L.lse + (size_t)B * Hq * Lq * 4);
  return L;
}

// Piece boundaries over U units (unit = one (batch, kv head) with its G query heads). pieces > 0:
// that many near-equal pieces (at most U). pieces == 0: three quarters in three equal pieces and
// the last quarter in two halves, so the last kernel and its output copy (the drain after the
// last input copy) are short while the first pieces stay large enough to keep the copies busy.
int host_pieces(long long U, int pieces, long long* bounds) {
  int n = 0;
  bounds[0] = 0;
  if (pieces > 0) {
    n = (int)std::min<long long>(pieces, U);
    for (int i = 1; i <= n; ++i) bounds[i] = U * i / n;
    return n;
  }
  const long long qtr = (U + 3) / 4;
  long long at = 0;
  for (int i = 0; i < 3 && at < U; ++i) {
    at = std::min(U, at + qtr);
    bounds[++n] = at;
  }
  const long long rest = U - at;
  if (rest > 1) bounds[++n] = at + (rest + 1) / 2;
  if (rest > 0) bounds[++n] = U;
  return n;
}

}  // namespace

extern "C" {

size_t attn_fwd_host_scratch_size(int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || d < 1 || dv < 1 || Hq % Hkv != 0) return 0;
  return host_layout(B, Hq, Hkv, Lq, Lk, d, dv).total;
}

attn_status attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host, float* lse_host,
                          int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, float scale, int causal, int dtype,
                          void* scratch, size_t scratch_bytes, int pieces, void* stream) {
  if (!valid_dtype(dtype)) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_common(q_host, k_host, v_host, o_host, lse_host, B, Hq, Hkv, Lq, Lk, d, dv, scale, causal);
  if (st != ATTN_OK) return st;
  if (d != dv || (d != 64 && d != 128)) return ATTN_ERR_UNSUPPORTED;
  if (pieces < 0 || pieces > kHostMaxPieces) return ATTN_ERR_INVALID_ARG;
  const HostLayout L = host_layout(B, Hq, Hkv, Lq, Lk, d, dv);
  if (!scratch || scratch_bytes < L.total || !aligned(scratch, 256)) return ATTN_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  HostPipe& hp = g_host_pipe[dev];
  std::lock_guard<std::mutex> lock(hp.mu);
  if (!host_pipe_init(hp)) return ATTN_ERR_CUDA;

  const int G = Hq / Hkv;
  const long long U = (long long)B * Hkv;
  long long bounds[kHostMaxPieces + 1];
  const int n = host_pieces(U, pieces, bounds);
  // bytes per unit of each tensor; a range of units is a contiguous range of every tensor
  const size_t uq = (size_t)G * Lq * d * 2, uk = (size_t)Lk * d * 2, uv = (size_t)Lk * dv * 2;
  const size_t uo = (size_t)G * Lq * dv * 2, ul = (size_t)G * Lq * 4;
  uint8_t* base = reinterpret_cast<uint8_t*>(scratch);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  auto H2D = cudaMemcpyHostToDevice;
  auto D2H = cudaMemcpyDeviceToHost;

  // the copies start after earlier work on the caller's stream (e.g. a previous call's kernels,
  // which read the same scratch)
  if (cudaEventRecord(hp.e_entry, cs) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamWaitEvent(hp.s_in, hp.e_entry, 0) != cudaSuccess) return ATTN_ERR_CUDA;
  for (int i = 0; i < n; ++i) {
    const long long u0 = bounds[i], nu = bounds[i + 1] - bounds[i];
    const uint8_t* qh = reinterpret_cast<const uint8_t*>(q_host);
    const uint8_t* kh = reinterpret_cast<const uint8_t*>(k_host);
    const uint8_t* vh = reinterpret_cast<const uint8_t*>(v_host);
    if (cudaMemcpyAsync(base + L.q + u0 * uq, qh + u0 * uq, nu * uq, H2D, hp.s_in) != cudaSuccess ||
        cudaMemcpyAsync(base + L.k + u0 * uk, kh + u0 * uk, nu * uk, H2D, hp.s_in) != cudaSuccess ||
        cudaMemcpyAsync(base + L.v + u0 * uv, vh + u0 * uv, nu * uv, H2D, hp.s_in) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaEventRecord(hp.e_in[i], hp.s_in) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaStreamWaitEvent(cs, hp.e_in[i], 0) != cudaSuccess) return ATTN_ERR_CUDA;
    // the piece is an attention problem of its own: nu "batches" of one kv head and G query heads
    st = with_elem(dtype, [&](auto e) {
      return fwd_impl<decltype(e), false>(base + L.q + u0 * uq, base + L.k + u0 * uk, base + L.v + u0 * uv,
                                          base + L.o + u0 * uo, reinterpret_cast<float*>(base + L.lse + u0 * ul),
                                          (int)nu, G, 1, Lq, Lk, d, scale, causal, SparseBlocks{nullptr, nullptr, 0},
                                          stream);
    });
    if (st != ATTN_OK) return st;
    if (cudaEventRecord(hp.e_run[i], cs) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaStreamWaitEvent(hp.s_out, hp.e_run[i], 0) != cudaSuccess) return ATTN_ERR_CUDA;
    uint8_t* oh = reinterpret_cast<uint8_t*>(o_host);
    if (cudaMemcpyAsync(oh + u0 * uo, base + L.o + u0 * uo, nu * uo, D2H, hp.s_out) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (lse_host) {
      uint8_t* lh = reinterpret_cast<uint8_t*>(lse_host);
      if (cudaMemcpyAsync(lh + u0 * ul, base + L.lse + u0 * ul, nu * ul, D2H, hp.s_out) != cudaSuccess)
        return ATTN_ERR_CUDA;
    }
  }
  // the caller's stream is ordered after the last output copy
  if (cudaEventRecord(hp.e_done, hp.s_out) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamWaitEvent(cs, hp.e_done, 0) != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

attn_status attn_check_device(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int word = 0, input_word = 0;
  if (cudaMemcpyFromSymbol(&word, attn::g_attn_dev_error, sizeof(word)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&input_word, attn::g_attn_dev_input_error, sizeof(input_word)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const unsigned int zero = 0;
  if (word != 0 && cudaMemcpyToSymbol(attn::g_attn_dev_error, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (input_word != 0 && cudaMemcpyToSymbol(attn::g_attn_dev_input_error, &zero, sizeof(zero)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (word != 0) return ATTN_ERR_TIMEOUT;
  if (input_word != 0) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

}  // extern "C"
