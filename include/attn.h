/*
 * attn.h -- C ABI of libattn_b200.so: exact scaled-dot-product attention on NVIDIA B200
 * (sm_100a).
 *
 *   O = softmax(scale * Q.K^T [+ causal mask]) . V,   LSE = ln sum_j exp(scale * q_i.k_j)
 *
 * The operation is the standard attention flow S = Q.K^T, P = softmax(S), O = P.V of the
 * FlashMLA-ETAP technical summary (gist.science 2506.01969, section "Mecanismo Central",
 * item 1). It is computed tile by tile in on-chip memory with a running-max / running-sum
 * softmax, so S and P never reach device memory (the "tiling" approach described in
 * "Activar Flash Attention con llama.cpp", section "Que es Flash Attention"). Key/value heads
 * may be shared by groups of query heads (GQA; same page, FAQ on GQA).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers named q, k, v, o, lse, o_part, lse_part, workspace, scratch are DEVICE pointers
 *    owned by the caller (names ending in _host are host pointers). The library allocates no
 *    device memory, never synchronises, and returns as soon as the work is enqueued on `stream`
 *    (a cudaStream_t passed as void*; NULL = legacy default stream).
 *  - Layouts are row-major and contiguous:
 *        q   [B, Hq,  Lq, d]   bf16 (or fp16, see the *_typed entry points)
 *        k   [B, Hkv, Lk, d]   same element type as q
 *        v   [B, Hkv, Lk, ldv] same element type, the first dv columns of each row are used
 *        o   [B, Hq,  Lq, dv]  same element type
 *        lse [B, Hq,  Lq]      fp32 (may be NULL)
 *  - GQA: query head h reads kv head h / (Hq / Hkv); Hq must be a multiple of Hkv.
 *  - Causal masking is bottom-right aligned: key j is visible to query row i iff
 *    j <= i + (Lk - Lq), i.e. the Lq queries are the last Lq positions of the sequence.
 *    causal != 0 with Lq > Lk is rejected (some rows would see no key).
 *  - LSE is the natural logarithm of sum_j exp(scale * q_i . k_j) over the visible keys.
 *  - Arithmetic: 16-bit inputs (bf16 by default), fp32 accumulation on the tensor cores, fp32
 *    softmax, P rounded to the input type before P.V, O rounded to the input type
 *    (round-to-nearest-even) at the end.
 *  - Errors: argument checks run on the host before any launch and return a non-zero status
 *    with nothing enqueued. A failed launch returns ATTN_ERR_CUDA. Kernels bound every wait
 *    on the GPU; a wait that runs out records ATTN_ERR_TIMEOUT in a device-side word that
 *    attn_check_device() reads (and clears); the kernel then stops early without hanging.
 *    Device-side index lists (attn_fwd_sparse_typed) that break their contract are recorded in
 *    a second device word (the kernel still finishes) and reported as ATTN_ERR_INVALID_ARG.
 *  - Thread safety: entry points keep no host state between calls except once-per-process
 *    lookups (the driver's tensor-map encoder, the resident-cluster count of a kernel) and the
 *    per-device state named at attn_fwd_host and attn_decode_noalloc; concurrent calls on
 *    different streams are safe.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1, /* NULL pointer, non-positive size, Hq % Hkv, causal Lq > Lk */
    ATTN_ERR_UNSUPPORTED = 2, /* valid attention, but a shape the library has no kernel for  */
    ATTN_ERR_MISALIGNED = 3,  /* a pointer or row stride breaks the 16-byte rule of TMA      */
    ATTN_ERR_WORKSPACE = 4,   /* decode workspace NULL or smaller than required             */
    ATTN_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed                        */
    ATTN_ERR_TIMEOUT = 6      /* a bounded wait inside a kernel ran out (see check_device)  */
} attn_status;

/*
 * Element type of q, k, v and o for the *_typed entry points. The untyped entry points take
 * bf16. FP16 is the input type of the FlashMLA-ETAP summary's measurements (H20, 148 TFLOPS
 * FP16, "Planteamiento del Problema"); both types run the same kernels, only the tensor-core
 * operand format, the TMA element type and the rounding of P and O change. FP16 keeps 10
 * mantissa bits but overflows above 65504: P lies in [0, 1] and O is a convex combination of V
 * rows, so neither can overflow when q, k and v are finite fp16 values.
 */
typedef enum {
    ATTN_DTYPE_BF16 = 0,
    ATTN_DTYPE_F16 = 1
} attn_dtype;

/*
 * attn_fwd -- prefill / general forward attention.
 *
 * Computes O and (optionally) LSE for all B*Hq*Lq query rows against Lk keys. V is dense:
 * its row stride equals dv.
 *   scale   multiplies Q.K^T (usually 1/sqrt(d)); must be finite and > 0.
 *   causal  0 = full attention, non-zero = bottom-right causal mask.
 * Supported: d == dv, d in {64, 128}; any B, Hq, Hkv (Hq % Hkv == 0), Lq, Lk >= 1.
 * Kernel: persistent warp-specialised tcgen05/TMEM kernel with TMA loads; two 128-row query
 * tiles per CTA ping-pong between two softmax warpgroups and one MMA-issuing thread.
 * Alignment: q, k, v, o 16-byte aligned (row strides are multiples of 16 bytes by shape).
 */
attn_status attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                     int Hq, int Hkv, int Lq, int Lk, int d, int dv, float scale, int causal,
                     void *stream);

/* attn_fwd for element type `dtype` (an attn_dtype); ATTN_ERR_INVALID_ARG for another value. */
attn_status attn_fwd_typed(const void *q, const void *k, const void *v, void *o, float *lse,
                           int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, float scale,
                           int causal, int dtype, void *stream);

/*
 * attn_fwd_host -- attn_fwd_typed on HOST buffers: the inputs are copied to the device, the
 * attention is computed and O and LSE are copied back, all enqueued asynchronously.
 *
 * The (batch, kv head) grid is cut into pieces of consecutive units (a unit is one kv head of
 * one batch with its Hq/Hkv query heads; a run of units is a contiguous range of q, k, v, o and
 * lse, so each piece is one copy per tensor and one attn_fwd call of its own). Piece i is copied
 * in on a library-owned stream, computed on `stream` and copied out on a second library-owned
 * stream, so the host-to-device copies, the kernels and the device-to-host copies of different
 * pieces overlap. The copies go over the host link, which is the bound of this call.
 *   q_host, k_host, v_host   HOST inputs in the layouts of attn_fwd; page-locked (pinned) memory
 *                           is needed for the copies to overlap (pageable memory works but the
 *                           copies then serialise).
 *   o_host, lse_host         HOST outputs (lse_host may be NULL); valid once `stream` has
 *                           completed the call (e.g. after cudaStreamSynchronize(stream)).
 *   scratch                  DEVICE buffer owned by the caller, 256-byte aligned, at least
 *                           attn_fwd_host_scratch_size(...) bytes: the device copies of q, k, v,
 *                           o and lse. Its contents on entry do not matter.
 *   pieces                   0: the library's split (three equal pieces over three quarters of
 *                           the units, the last quarter in two halves, so that the drain after
 *                           the last input copy is short); 1..64: that many near-equal pieces
 *                           (fewer if there are fewer units).
 * The call is ordered after earlier work on `stream`, and later work on `stream` is ordered
 * after its last copy. The library creates its two copy streams and its events on the first call
 * on each device and keeps them until the process exits (they hold no device memory); concurrent
 * calls on one device enqueue one after the other. Other arguments, checks and supported shapes
 * are those of attn_fwd_typed; a scratch that is NULL, too small or misaligned gives
 * ATTN_ERR_WORKSPACE.
 */
size_t attn_fwd_host_scratch_size(int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv);
attn_status attn_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host,
                          float *lse_host, int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv,
                          float scale, int causal, int dtype, void *scratch, size_t scratch_bytes,
                          int pieces, void *stream);

/*
 * attn_fwd_sparse_typed -- block-sparse forward attention over caller-given index lists.
 *
 * The MInference article (7minutos.es, on sparse attention for long-context prefill) describes
 * attention weights that concentrate on a few structured regions (A-shape, vertical bars,
 * sparse blocks) and a prefill that computes only those regions from an index built per input.
 * This entry point takes such an index as given (building it is not part of this library) and
 * computes the exact softmax attention restricted to it:
 *   query rows are cut into blocks of 128 rows, keys into blocks of 128 keys; query block qb of
 *   head (b, h) sees the keys of the blocks listed in
 *       block_idx[((b * Hq + h) * nqb + qb) * max_blocks + t],  t < block_cnt[(b * Hq + h) * nqb + qb]
 *   (nqb = ceil(Lq / 128)), intersected with the causal mask when causal != 0. Each list must be
 *   strictly increasing with entries in [0, ceil(Lk / 128)); entries past the count are ignored.
 *   A row that sees no key gets O = 0 and LSE = -inf. An A-shape pattern is the list {0} plus
 *   the blocks of a local window; block-sparse patterns list their blocks directly.
 *   block_idx, block_cnt  DEVICE int32 arrays owned by the caller, 4-byte aligned, read-only.
 * Other arguments, layouts and supported shapes are those of attn_fwd_typed. A list that breaks
 * its contract is read up to the offending entry (the kernel completes on the truncated list and
 * nothing outside the arrays is read) and recorded on the device: attn_check_device() then
 * returns ATTN_ERR_INVALID_ARG.
 */
attn_status attn_fwd_sparse_typed(const void *q, const void *k, const void *v, void *o, float *lse,
                                  int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv,
                                  float scale, int causal, const int32_t *block_idx,
                                  const int32_t *block_cnt, int max_blocks, int dtype,
                                  void *stream);

/*
 * attn_decode_workspace_size -- bytes of device workspace attn_decode needs for the given
 * shape and split count (num_splits = 0: the count attn_decode chooses on this device).
 * Layout of the workspace: o_part fp32 [num_splits, B*Hq*Lq, dv] followed (256-byte
 * aligned) by lse_part fp32 [num_splits, B*Hq*Lq]. Returns 0 for invalid sizes.
 * Hkv and Lk are arguments (a plain split count would need only B, Hq, Lq and dv) because with
 * num_splits = 0 the library plans the splits itself from the number of (batch, kv head) units
 * B*Hkv and the key length Lk: the balanced schedule cuts the B*Hkv*Lk keys into one run per SM
 * slot, and the partial count of a kv head follows from where those runs fall.
 */
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int dv,
                                  int num_splits);

/*
 * attn_decode -- split-KV decode attention for a few query tokens against a long KV cache.
 *
 * The Lk keys of every (batch, kv head) are cut into num_splits contiguous chunks processed
 * by different CTAs. Each chunk writes a partial O (fp32, already divided by its own softmax
 * sum) and a partial LSE (-inf for a chunk without visible keys) into the workspace; an
 * attn_combine launch on the same stream then merges them into O (bf16) and LSE (fp32).
 *
 *   v, ldv   V rows with stride ldv >= dv. MLA latent KV passes v == k and ldv == d: V is the
 *            first dv columns of each latent K row, and every row is read from memory once.
 *   num_splits  1..256: every (batch, kv head) is cut into that many equal chunks. 0: the library's
 *               schedule. For the queries-on-M kernel that is a balanced grid of one CTA per SM
 *               slot, each taking an equal run of consecutive keys of the (batch * Hkv + kv head,
 *               key) sequence (a run may end in one kv head and continue in the next), so every SM
 *               streams the same number of bytes; a kv head then gets up to
 *               attn_decode_default_splits(...) partials. Other kernels use equal chunks with a
 *               count chosen from the shape and the SM count.
 *   workspace   device buffer of at least attn_decode_workspace_size(...) bytes, 256-byte
 *               aligned. Its contents on entry do not matter.
 * Supported: rows per kv head R = (Hq/Hkv)*Lq <= 64; d <= 576, dv <= 512, d and dv
 * multiples of 8 (16-byte rows). Two tensor-core kernels serve R <= 32:
 *   - query rows on the MMA M dimension (padded to 64), keys on N: latent KV (v == k, ldv == d,
 *     d % 64 == 0, dv % 128 == 0, dv <= d) or a dense V with dv == d in {128, 256}; this is the
 *     kernel attn_decode uses (measured fastest on B200);
 *   - key length on M (the transposed flow of the FlashMLA-ETAP summary, "Mecanismo Central",
 *     items 1-3): latent KV only, selectable through attn_decode_ex.
 * Other shapes use a CUDA-core kernel.
 */
attn_status attn_decode(const void *q, const void *k, const void *v, void *o, float *lse,
                        int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, int ldv,
                        float scale, int causal, int num_splits, void *workspace,
                        size_t workspace_bytes, void *stream);

/* Decode kernels selectable through attn_decode_ex (attn_decode uses ATTN_DECODE_AUTO). */
typedef enum {
    ATTN_DECODE_AUTO = 0,      /* tensor-core kernel when the shape allows it, else CUDA cores */
    ATTN_DECODE_CUDA_CORE = 1, /* fp32 FMA dot products, any supported shape                   */
    ATTN_DECODE_TCGEN05_T = 2, /* tcgen05, key length on M (transposed flow)                   */
    ATTN_DECODE_TCGEN05_N = 3  /* tcgen05, query rows on M (padded to 64), keys on N            */
} attn_decode_impl;

/* attn_decode with an explicit kernel choice (for measurement); ATTN_ERR_UNSUPPORTED if the
 * requested kernel cannot run the shape. Other arguments as attn_decode. */
attn_status attn_decode_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                           int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, int ldv,
                           float scale, int causal, int num_splits, void *workspace,
                           size_t workspace_bytes, int impl, void *stream);

/* attn_decode_ex for element type `dtype` (an attn_dtype); ATTN_ERR_INVALID_ARG for another
 * value. The workspace partials are fp32 whatever the element type. */
attn_status attn_decode_typed(const void *q, const void *k, const void *v, void *o, float *lse,
                              int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, int ldv,
                              float scale, int causal, int num_splits, void *workspace,
                              size_t workspace_bytes, int impl, int dtype, void *stream);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device memory.
 *
 * No counterpart in the pages; this is an interface addition. Some callers cannot call
 * cudaMalloc or hand over a workspace: code that runs while a CUDA graph is being captured
 * elsewhere in the process, memory-capped serving processes with a fixed pool, or plugins that
 * only receive input and output pointers. This entry point takes the same arguments as
 * attn_decode minus the workspace and keeps the split partials in a scratch array compiled
 * into the library: ATTN_DECODE_NOALLOC_SCRATCH_BYTES bytes of device memory that every GPU
 * which loads the library holds until the process exits. It calls no allocating routine.
 *   - Shapes whose partials (attn_decode_workspace_size for the chosen split count) exceed
 *     the scratch size are rejected with ATTN_ERR_WORKSPACE before anything is enqueued; pass a
 *     smaller num_splits or use attn_decode with a caller workspace.
 *   - The first call on each device looks up the device address of the scratch array (a
 *     synchronous host call that may load the library's GPU code). Make that first call before
 *     any stream capture on that device. The address is kept per device together with the id
 *     of the CUDA context it belongs to; after a cudaDeviceReset (a new context) the next call
 *     looks it up again, so that call too must come before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents. The kernels write
 *     every scratch byte they later read, so nothing needs clearing between calls, but two
 *     calls that overlap on the GPU (different streams, no ordering between them) race on the
 *     array and give wrong results. Order such calls on one stream or with events.
 * Other arguments, supported shapes and kernel choice are those of attn_decode.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)
attn_status attn_decode_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, int ldv,
                                float scale, int causal, int num_splits, void *stream);

/*
 * attn_combine -- log-sum-exp merge of split partials over disjoint key ranges. Flash attention
 * updates its softmax statistics "iteratively and locally", block by block ("Activar Flash
 * Attention con llama.cpp", section "Que es Flash Attention"); merging the (max, sum, output)
 * of two key chunks is that same update applied once more, written here with the log-sum-exp
 * of each chunk:
 *   LSE = ln sum_s exp(lse_s),  O = sum_s exp(lse_s - LSE) * O_s   (splits with lse_s = -inf
 *   carry no weight). o_part fp32 [num_splits, rows, dv], lse_part fp32 [num_splits, rows],
 *   rows = B*Hq*Lq in [B, Hq, Lq] order; o bf16 [rows, dv]; lse fp32 [rows] (may be NULL).
 * A row whose every split is empty gets O = 0 and LSE = -inf.
 */
attn_status attn_combine(const float *o_part, const float *lse_part, void *o, float *lse,
                         int B, int Hq, int Lq, int dv, int num_splits, void *stream);

/* attn_combine writing o in element type `dtype` (an attn_dtype). */
attn_status attn_combine_typed(const float *o_part, const float *lse_part, void *o, float *lse,
                               int B, int Hq, int Lq, int dv, int num_splits, int dtype,
                               void *stream);

/* Number of partial results per (batch, kv head) that attn_decode uses with num_splits = 0 on the
 * current device (the most any kv head gets under the balanced schedule) for a call with these
 * sizes. latent != 0: MLA latent KV (v == k, ldv == d, V the first dv columns of each K row);
 * latent == 0: a separate dense V. Returns 0 for invalid sizes. */
int attn_decode_default_splits(int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv, int latent);

/*
 * attn_check_device -- synchronises `stream`, then reads and clears the device-side error
 * word that kernels set when a bounded wait runs out or a device index list is invalid. Returns
 * ATTN_OK, ATTN_ERR_TIMEOUT, ATTN_ERR_INVALID_ARG (bad index list) or ATTN_ERR_CUDA (a sticky
 * CUDA error from earlier work). For tests and diagnostics; the
 * compute entry points never synchronise.
 */
attn_status attn_check_device(void *stream);

/* Static, human-readable name of a status code. */
const char *attn_status_string(attn_status status);

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
int attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
