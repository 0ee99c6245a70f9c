/*
 * kvq.h -- C ABI of the SRFT-int4 KV-cache library for NVIDIA B200 (sm_100a).
 *
 * The method is the fused KV-cache compression of "When Quantization Is Free:
 * An int4 KV Cache That Outruns fp16 on Apple Silicon" (arXiv 2605.05699):
 *   [ABS] paperdance.org/p/2605.05699, English abstract: one fused kernel does the whole
 *         encode -- a random-sign FFT, one factor per channel, one absolute-maximum
 *         scale per channel group, and two 4-bit codes packed into each byte.
 *   [M1]  gist.science/de/paper/2605.05699, "Methodik" 1: the rotation is the unitary
 *         DFT F applied after a fixed random +/-1 sign vector s, the complex result
 *         packed to real values.
 *   [M2]  same page, "Methodik" 2: the kernel's steps in order -- signs applied on
 *         load, the FFT butterflies, the Hermitian-symmetric spectrum unpacked to real
 *         values, the per-channel factor, the group abs-max and rounding to signed
 *         4-bit (or 8-bit) integers, and nibble packing.
 * The read path (decode, decode attention on the packed cache) is not on the
 * pages; it is the inverse transform and softmax attention taken in the rotated
 * domain, valid because F is unitary (<q, R^T y> = <R q, y>).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Element types are given by their bits: fp16 values are passed as uint16_t
 *    (IEEE binary16), codes as uint8_t. No CUDA or torch types appear here.
 *  - All data pointers are DEVICE pointers on the plan's device (the current
 *    device for kvq_attend_decode_ref), except where a comment says "host".
 *    The caller owns every buffer; no entry point allocates device memory
 *    except kvq_plan_create. All pointers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Every call is asynchronous on that stream and never synchronises.
 *  - Errors: arguments are checked on the host before anything is launched; a
 *    failed check returns a negative kvq_status and touches no memory. A CUDA
 *    error at launch returns KVQ_ERR_CUDA. kvq_last_error() gives a one-line
 *    description of the last failure on the calling thread.
 *  - Layouts (row-major, innermost last):
 *      x / out vectors   fp16 [B, H, n, D]
 *      codes cache       u8   [B, H, T_cap, D/2]   two's-complement nibbles,
 *                                                  channel 2j in the low nibble of byte j
 *                                                  (int8 plans, kvq_plan_create_ex:
 *                                                  [B, H, T_cap, D], one byte per channel;
 *                                                  every "D/2" below is then D)
 *      scales cache      fp16 [B, H, T_cap, D/G]   scale of channels [gG, gG+G)
 *      q                 fp16 [B, Hq, D]
 *      attention out     fp16 [B, Hq, D]
 *  - Rotated channel order: channel 0 = DC, channels 2k-1 / 2k = cos / sin of
 *    frequency k (k = 1 .. D/2-1), channel D-1 = Nyquist. Row 2k-1 of the real
 *    basis is sqrt(2/D) cos(2 pi k n / D), row 2k is sqrt(2/D) sin(2 pi k n / D).
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, bad sign/lambda value */
  KVQ_ERR_UNSUPPORTED = -2, /* head_dim not 128/256, group not 32/16, Hq % Hkv != 0   */
  KVQ_ERR_ALIGNMENT = -3,   /* pointer not 16-byte aligned, or T_cap odd (attention)   */
  KVQ_ERR_CAPACITY = -4,    /* pos + n > T_cap, t0 + n > T_cap, T_len > T_cap           */
  KVQ_ERR_CUDA = -5,        /* a CUDA runtime call or launch failed                    */
  KVQ_ERR_WORKSPACE = -6,   /* workspace missing or smaller than kvq_workspace_size    */
  KVQ_ERR_DEVICE = -7       /* no sm_100 device, or plan used on another device        */
} kvq_status;

/* Opaque per-(s, lambda) transform plan. Immutable after creation; one plan may be
 * used from several streams and host threads at once. */
typedef struct kvq_plan kvq_plan;

/* The rotation R of a plan: the SRFT of [M1], R = F_r diag(s) (the default), or the
 * SRHT the pages compare it with ([M1] "Begruendung" / "Ergebnis": equal quality),
 * read here as R = H diag(s) / sqrt(D), H the Sylvester Hadamard matrix in natural
 * order, H[i][j] = (-1)^popcount(i & j). */
typedef enum { KVQ_TRANSFORM_SRFT = 0, KVQ_TRANSFORM_SRHT = 1 } kvq_transform;

/*
 * kvq_plan_create -- [M1] fixes s, [M2] lambda (one factor per rotated channel); the
 * SRFT plan (kvq_plan_create_transform with KVQ_TRANSFORM_SRFT).
 *   out         host: receives the new plan.
 *   head_dim    D: 128 or 256.
 *   group       G: channels per abs-max scale group (32; 16 also accepted).
 *   signs_host  host int8[D], every entry +1 or -1 (the fixed random sign vector s).
 *   lambda_host host float[D], every entry finite and > 0 (per-channel lambda).
 * Allocates one device block on the current device, the plan's device: the
 * per-channel factors and sign masks derived from s and lambda, the tensor-core
 * encode's operand Lambda R as an fp16 hi/lo pair (2 D^2 halves) and the attention
 * kernels' 128-point transform (64 KB).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA, DEVICE.
 */
kvq_status kvq_plan_create(kvq_plan** out, int head_dim, int group, const int8_t* signs_host,
                           const float* lambda_host);

/* kvq_plan_create with the rotation chosen: transform is a kvq_transform value
 * (UNSUPPORTED otherwise). Every entry point accepts either kind; the two plans of
 * an attention call must use the same kind. */
kvq_status kvq_plan_create_transform(kvq_plan** out, int head_dim, int group, const int8_t* signs_host,
                                     const float* lambda_host, int transform);

/* The plan's kvq_transform value; -1 for a NULL plan. */
int kvq_plan_transform(const kvq_plan* plan);

/*
 * kvq_plan_create_ex -- kvq_plan_create_transform with the code width chosen ([M2]
 * rounds "to signed int4/int8"):
 *   bits  4: codes clamp(rint(y / scale), -7, 7) with scale = fp16_rn(min(absmax/7,
 *            65504)), two per byte (nibble pairs, as kvq_encode describes);
 *         8: the same with 127 in place of 7 (scale = fp16_rn(min(absmax/127, 65504)),
 *            codes in [-127, 127]), one two's-complement byte per channel, channel i at
 *            byte i. Every "D/2" code row below is then D bytes.
 *   Other values: UNSUPPORTED. int8 plans are served by both encode paths, decode and
 *   every attention entry point; both plans of an attention call, and all jobs of a
 *   batch, must share the code width.
 */
kvq_status kvq_plan_create_ex(kvq_plan** out, int head_dim, int group, const int8_t* signs_host,
                              const float* lambda_host, int transform, int bits);

/* The plan's code width (4 or 8); -1 for a NULL plan. */
int kvq_plan_bits(const kvq_plan* plan);

/* Frees the plan and its device block. Passing NULL is a no-op. The caller must
 * ensure no launch that uses the plan is still pending. */
kvq_status kvq_plan_destroy(kvq_plan* plan);

/* Plan properties (head_dim, group); -1 for a NULL plan. */
int kvq_plan_head_dim(const kvq_plan* plan);
int kvq_plan_group(const kvq_plan* plan);

/*
 * kvq_encode -- the fused encode of [ABS]/[M2]: for each fp16 vector x of
 * x[B, H, n, D]: y = lambda * (F_r . diag(s) . x) (fp32), then per group of G
 * rotated channels scale = fp16_rn(min(absmax/7, 65504)) and
 * c = clamp(rint(y / scale), -7, 7) (0 where scale == 0), nibble-packed.
 *   x        fp16 [B, H, n, D] contiguous.
 *   codes    u8   [B, H, T_cap, D/2]; rows pos .. pos+n-1 of every (b, h) are written.
 *   scales   fp16 [B, H, T_cap, D/G]; same rows written.
 *   T_cap    capacity (tokens) of the cache; pos + n <= T_cap.
 * No other cache row is touched. n == 0 is a no-op.
 * Errors: INVALID_ARG, ALIGNMENT, CAPACITY, DEVICE, CUDA.
 */
kvq_status kvq_encode(const kvq_plan* plan, const uint16_t* x, int B, int H, int n, uint8_t* codes,
                      uint16_t* scales, int T_cap, int pos, void* stream);

/*
 * kvq_encode_batch -- the same encode for many independent (plan, x, cache) jobs in
 * one grouped launch, e.g. K and V of every layer of a prefill (each with its own
 * s and lambda). Each job is exactly one kvq_encode call; jobs are processed in
 * any order and must not write overlapping cache rows.
 *   jobs    host array of njobs descriptors (read during the call only). All jobs
 *           with work must use plans of one head_dim, group and device. Jobs with
 *           B, H or n == 0 are skipped. Up to 64 jobs share one kernel launch.
 * Errors: as kvq_encode, reported for the first offending job; nothing is launched.
 */
typedef struct kvq_encode_job {
  const kvq_plan* plan;
  const uint16_t* x;   /* fp16 [B, H, n, D] */
  uint8_t* codes;      /* u8   [B, H, T_cap, D/2] */
  uint16_t* scales;    /* fp16 [B, H, T_cap, D/G] */
  int B, H, n, T_cap, pos;
} kvq_encode_job;

kvq_status kvq_encode_batch(const kvq_encode_job* jobs, int njobs, void* stream);

/*
 * kvq_set_encode_path / kvq_get_encode_path -- which kernel kvq_encode and
 * kvq_encode_batch run (process-wide setting; not on the pages):
 *   0  default: the dense tensor-core encode (path 2) where it exists;
 *   1  always the register-FFT encode (one radix-2 real FFT per vector in registers);
 *   2  the dense tensor-core encode (tcgen05 GEMM against W = Lambda F_r diag(s) held
 *      as an fp16 hi + lo pair; for SRHT plans the exact W = H diag(s)), head_dim 128
 *      and 256 with group 32 or 16;
 *   3  the radix-2 split on the tensor cores: the two 128-point real DFTs of the even
 *      and odd samples as products against the plan-independent F128 (fp16 hi + lo),
 *      joined by one radix-2 step (half the tensor work of path 2); head_dim 256 SRFT
 *      plans only (KVQ_ERR_UNSUPPORTED otherwise).
 * Both produce codes and scales that meet the same acceptance rule against the
 * fp64 definition; they may differ from each other only at rounding boundaries.
 * Set it between launches, not while another thread is encoding.
 * Errors: INVALID_ARG for a value other than 0, 1, 2, 3.
 */
kvq_status kvq_set_encode_path(int path);
int kvq_get_encode_path(void);

/*
 * kvq_decode -- the inverse: x_hat = diag(s) . F_r^T . (c * scale / lambda), rounded
 * to fp16, for cache rows t0 .. t0+n-1 of every (b, h). The encode's definition
 * ("When Quantization Is Free", gist.science/de/paper/2605.05699, "Methodik" 1-2) is
 * a linear map up to the quantiser, so this is its exact inverse applied to the
 * dequantised values (the pages describe no decode kernel; this one follows from that
 * definition).
 *   codes, scales  the cache as written by kvq_encode (device, 16-byte aligned);
 *   out  fp16 [B, H, n, D] contiguous (device, 16-byte aligned), written, never read.
 * Default kernel (kvq_set_decode_path): the tensor-core product against the plan's fp16
 * decode matrix, within 5e-4 relative L2 of the fp64 result per vector (the fp16 output
 * alone rounds at 2^-11 relative); path 1 runs the register inverse FFT in fp32.
 * Errors: INVALID_ARG, ALIGNMENT, CAPACITY, DEVICE, CUDA.
 */
kvq_status kvq_decode(const kvq_plan* plan, const uint8_t* codes, const uint16_t* scales, int B,
                      int H, int T_cap, int t0, int n, uint16_t* out, void* stream);

/*
 * kvq_set_decode_path / kvq_get_decode_path -- which kernel kvq_decode runs
 * (process-wide setting; not on the pages):
 *   0  default: tensor cores -- the codes dequantised to fp16 (code times the group
 *      scale, normalised per vector by a power of two), one tcgen05 product against
 *      W_dec = diag(s) Q^T Lambda^-1 in fp16 (built with the plan), fp32 accumulation;
 *   1  the register inverse FFT (SRFT) or Walsh-Hadamard butterflies (SRHT) in fp32.
 * Both serve every plan (head_dim 128 / 256, group 32 / 16, int4 / int8, SRFT / SRHT).
 * Set it between launches, not while another thread is decoding.
 * Errors: INVALID_ARG for a value other than 0, 1.
 */
kvq_status kvq_set_decode_path(int path);
int kvq_get_decode_path(void);

/*
 * kvq_workspace_size -- bytes of device workspace that kvq_attend_decode and
 * kvq_attend_decode_ref need for these shapes (T_cap = the cache capacity; the
 * split of the sequence is chosen from it). The workspace holds the per-split
 * softmax partials and one completion counter per (b, kv head, head tile).
 * The counters must be zero before the first call that uses a workspace (e.g.
 * cudaMemsetAsync once after allocation); every completed call leaves them zero
 * again. Two calls must not use the same workspace concurrently.
 */
size_t kvq_workspace_size(int B, int Hq, int Hkv, int head_dim, int T_cap);

/*
 * kvq_attend_decode -- one-query decode attention read straight from the packed
 * int4 K/V cache, in the rotated domain (not on the pages; follows from [M1]):
 *   q_t = Lambda_K^-1 R_K q (fp32, kept as an fp16 hi + lo pair),
 *   score_t = sigma * sum_g scaleK[t,g] * sum_{i in g} q_t[i] * cK[t,i],
 *   o_t = sum_t softmax(score)_t * (cV[t] * scaleV[t]) (split over the sequence,
 *         combined with the log-sum-exp rule),
 *   out = diag(s_V) F_r^T Lambda_V^-1 o_t  -> fp16.
 *   pk, pv     plans of the K and V transforms (same head_dim and group).
 *   q          fp16 [B, Hq, D]; query head h reads KV head h / (Hq / Hkv).
 *   k_codes, v_codes    u8 [B, Hkv, T_cap, D/2];  k_scales, v_scales fp16 [B, Hkv, T_cap, D/G].
 *   seq_lens   device int32[B] (tokens 0 .. seq_lens[b]-1 are attended; values are
 *              clamped to [0, T_cap]), or NULL to use T_len for every batch entry.
 *   softmax_scale  sigma; <= 0 selects 1/sqrt(D).
 *   out        fp16 [B, Hq, D]. A batch entry with no tokens gets zeros.
 *   workspace  device buffer of >= kvq_workspace_size(B, Hq, Hkv, D, T_cap) bytes.
 * T_cap must be even (the scale rows are fetched by TMA in 16-byte units).
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CAPACITY, WORKSPACE, DEVICE, CUDA.
 */
kvq_status kvq_attend_decode(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q,
                             const uint8_t* k_codes, const uint16_t* k_scales,
                             const uint8_t* v_codes, const uint16_t* v_scales, int B, int Hq,
                             int Hkv, int T_cap, const int32_t* seq_lens, int T_len,
                             float softmax_scale, uint16_t* out, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * kvq_attend_decode_append -- one decode step of one layer in one launch: the new
 * token's K and V rows are encoded into the caches at token `pos` (exactly what
 * kvq_encode with n = 1 at `pos` stores, up to fp32 rounding of the transform: a
 * code may differ only where the pre-rounding value lies at a rounding boundary),
 * and the query attends over tokens 0 .. pos, the new one included, as
 * kvq_attend_decode with T_len = pos + 1. The new token's encode is folded into the
 * attention launch; the pages run the same fused encode for a decoded token as for a
 * prefill, [M2].
 *   k_new, v_new   fp16 [B, Hkv, D], the new token's rows (original domain).
 *   k_codes, k_scales, v_codes, v_scales   the caches as in kvq_attend_decode,
 *              written at token pos (every (b, kv head)), read at tokens < pos.
 *   pos        0 <= pos < T_cap, the same for every batch entry.
 *   q, out, softmax_scale, workspace   as in kvq_attend_decode.
 * The other tokens of the caches are only read. Errors: as kvq_attend_decode;
 * CAPACITY when pos >= T_cap.
 */
kvq_status kvq_attend_decode_append(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q,
                                    const uint16_t* k_new, const uint16_t* v_new, uint8_t* k_codes,
                                    uint16_t* k_scales, uint8_t* v_codes, uint16_t* v_scales, int B,
                                    int Hq, int Hkv, int T_cap, int pos, float softmax_scale,
                                    uint16_t* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * kvq_attend_decode_partial -- sequence-sharded (context-parallel) decode, step 1: the
 * attention of kvq_attend_decode over cached tokens t_begin .. t_end - 1 only, left as
 * each query head's softmax partial in the rotated domain instead of an output (a GPU
 * holding one slice of a long context attends over its slice; the slices' partials are
 * exchanged, e.g. by an all-gather, and merged by kvq_attend_combine). Not on the pages.
 *   partial   fp32 [B, Hq, D + 4]: per query head m (the maximum of the scores, in
 *             base-2 units of softmax_scale * score), l (sum of 2^(score - m)), two pad
 *             floats, o_t[D] = sum 2^(score - m) cV * scaleV (rotated domain, not
 *             normalised). A head with no tokens gets m = -inf, l = 0, o_t = 0.
 *   t_begin   even, 0 <= t_begin <= t_end <= T_cap; the same range for every batch entry.
 *   other arguments as kvq_attend_decode (no seq_lens).
 * Errors: as kvq_attend_decode.
 */
kvq_status kvq_attend_decode_partial(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q,
                                     const uint8_t* k_codes, const uint16_t* k_scales,
                                     const uint8_t* v_codes, const uint16_t* v_scales, int B, int Hq,
                                     int Hkv, int T_cap, int t_begin, int t_end, float softmax_scale,
                                     float* partial, void* workspace, size_t ws_bytes, void* stream);

/*
 * kvq_attend_combine -- step 2: merges n_parts partials of the same query heads (fp32
 * [n_parts, B, Hq, D + 4], e.g. gathered from the GPUs of a context-parallel group) by
 * the log-sum-exp rule, M = max m_r, L = sum l_r 2^(m_r - M), O = sum o_r 2^(m_r - M),
 * and un-rotates O / L with the V plan: the result equals kvq_attend_decode over the
 * union of the ranges up to fp32 rounding. 1 <= n_parts <= 64.
 *   out   fp16 [B, Hq, D]. Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, DEVICE, CUDA.
 */
kvq_status kvq_attend_combine(const kvq_plan* pv, const float* partials, int n_parts, int B, int Hq,
                              uint16_t* out, void* stream);

/*
 * kvq_attend_decode_batch -- kvq_attend_decode for many independent problems of one
 * shape in one grouped launch (up to 32 per launch; more are run as consecutive
 * launches on the stream), e.g. the decode attention of every layer of a model
 * step when the layers' queries are already known, or several caches of one
 * shape. Each job is exactly one kvq_attend_decode call with the shared sizes.
 *   jobs     host array of njobs descriptors (read during the call only). All plans
 *            share one head_dim, group (32) and device.
 *   B, Hq, Hkv, T_cap, seq_lens, T_len, softmax_scale   shared by every job.
 *   workspace  >= kvq_workspace_size(min(njobs, 32) * B, Hq, Hkv, D, T_cap) bytes,
 *            counters zero before the first use (every call leaves them zero).
 * Errors: as kvq_attend_decode, reported for the first offending job; nothing is
 * launched when any job fails validation.
 */
typedef struct kvq_attend_job {
  const kvq_plan* pk;        /* K plan */
  const kvq_plan* pv;        /* V plan */
  const uint16_t* q;         /* fp16 [B, Hq, D] */
  const uint8_t* k_codes;    /* u8   [B, Hkv, T_cap, D/2] */
  const uint16_t* k_scales;  /* fp16 [B, Hkv, T_cap, D/32] */
  const uint8_t* v_codes;
  const uint16_t* v_scales;
  uint16_t* out;             /* fp16 [B, Hq, D] */
} kvq_attend_job;

kvq_status kvq_attend_decode_batch(const kvq_attend_job* jobs, int njobs, int B, int Hq, int Hkv,
                                   int T_cap, const int32_t* seq_lens, int T_len,
                                   float softmax_scale, void* workspace, size_t ws_bytes,
                                   void* stream);

/*
 * kvq_attend_decode_noalloc -- kvq_attend_decode for callers that cannot allocate
 * device memory: a serving runtime whose memory is planned up front, code that
 * runs while a stream is being captured (cudaMalloc is not allowed there), or a
 * host where another component owns the allocator. The paper has no counterpart;
 * this is a library convenience.
 * Same arguments and results as kvq_attend_decode, without the workspace: the
 * scratch is one file-scope device array of 8 MiB inside the library (every GPU
 * that loads the library holds it until the process exits). Shapes whose split
 * needs more than 8 MiB of scratch are rejected with KVQ_ERR_WORKSPACE before
 * anything is launched (use kvq_attend_decode for those).
 * No cudaMalloc, cudaFree or allocating library call is made. The first call on
 * a device looks up the array's device address (cudaGetSymbolAddress with that
 * device current); make that first call before any stream capture. Each call
 * clears the array's counters with a stream-ordered memset before its kernels.
 * All calls share the one array and it keeps the last call's contents, so calls
 * whose executions overlap on the GPU (other streams, other host threads, or
 * graph branches) race and must be serialised by the caller.
 * Errors: as kvq_attend_decode.
 */
kvq_status kvq_attend_decode_noalloc(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q,
                                     const uint8_t* k_codes, const uint16_t* k_scales,
                                     const uint8_t* v_codes, const uint16_t* v_scales, int B, int Hq,
                                     int Hkv, int T_cap, const int32_t* seq_lens, int T_len,
                                     float softmax_scale, uint16_t* out, void* stream);

/*
 * kvq_attend_decode_ref -- the fp16-cache comparator for the same shapes: the same
 * split-sequence softmax attention over fp16 K/V [B, Hkv, T_cap, D] with no
 * rotation. This is the uncompressed baseline the int4 path is measured against
 * (the pages compare int4 with an fp16 cache, [ABS]).
 * Same argument rules as kvq_attend_decode (head_dim = D is 128 or 256).
 */
kvq_status kvq_attend_decode_ref(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B,
                                 int Hq, int Hkv, int head_dim, int T_cap,
                                 const int32_t* seq_lens, int T_len, float softmax_scale,
                                 uint16_t* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * kvq_attend_split_info -- the sequence split the attention entry points choose for
 * these shapes on the current device (not on the pages; a planning query, e.g. to
 * size buffers or to check which merge path a call takes). One unit is one (batch
 * entry, kv head, tile of up to 8 query heads); its tokens are cut into *splits
 * contiguous ranges, one CTA each; groups of *cluster CTAs merge their softmax
 * partials through distributed shared memory, and a unit with *splits / *cluster > 1
 * also merges its cluster partials through the workspace.
 *   B, Hq, Hkv, head_dim   as in kvq_attend_decode (one problem, not a batch of jobs).
 *   group, bits   the plans' group (32 or 16) and code width (4 or 8); bits = 16 asks
 *                 for kvq_attend_decode_ref's fp16 kernel (group ignored).
 *   T             the token count the split is chosen from: T_cap when seq_lens is
 *                 passed, else T_len (kvq_attend_decode_append: pos; _partial:
 *                 t_end - t_begin).
 *   splits, cluster, head_tiles   host outputs; any may be NULL.
 * Errors: INVALID_ARG, UNSUPPORTED, DEVICE (no sm_100 device current).
 */
kvq_status kvq_attend_split_info(int B, int Hq, int Hkv, int head_dim, int group, int bits, int T,
                                 int* splits, int* cluster, int* head_tiles);

/*
 * kvq_debug_wait_timeout -- a self-test of the kernels' failure path (not on the
 * pages): launches one CTA on `stream` that waits, through the same bounded wait the
 * kernels use, on an mbarrier that nothing will complete, with a budget of limit_us
 * microseconds (1 .. 1e6) instead of 1 s. When the budget runs out the CTA raises
 * flag 1 (the flag of a TMA load that never arrived) and exits; the context stays
 * usable. kvq_poll_device_errors then reports the flag. Errors: INVALID_ARG, DEVICE,
 * CUDA.
 */
kvq_status kvq_debug_wait_timeout(uint32_t limit_us, void* stream);

/*
 * kvq_poll_device_errors -- synchronises the current device, then returns (in
 * *flags, host, may be NULL) the bit flags raised by kernels of this library
 * since the last poll, and clears them: 1 = a kernel gave up waiting for a TMA
 * load (bounded wait of 1 s), 2 = a bulk store did not drain, 4 = an attention
 * cluster merge did not receive (or release) a partial within 1 s. 0 means none.
 * Errors: CUDA.
 */
kvq_status kvq_poll_device_errors(uint32_t* flags);

/* Static description of a status code. */
const char* kvq_status_string(kvq_status status);

/* One-line description of the last failed call on this host thread ("" if none). */
const char* kvq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
