/*
 * cvq.h -- C ABI of libcvq: CommVQ decode attention read directly from an additively
 * vector-quantized KV cache whose key codebook commutes with RoPE.
 *
 * The method (CommVQ review page, pith.science arXiv 2506.18879, "key_machinery";
 * CommVQ summary page, atlas.scime.ai, "Approach"): keys and values of the cache are
 * stored as uint8 code indices into small additive codebooks.  A key codeword is a
 * complex number c = a + ib per RoPE pair, i.e. the 2x2 block [[a,-b],[b,a]], which
 * commutes with every RoPE rotation, so the query side can be combined with the
 * codebook once per query and reused at every cached position.  Softmax weights are
 * accumulated per value code before the value codebook multiply (review page,
 * "forward_implications", 4th item).
 *
 * Two instances (cvq_shape.group_dim), both with head_dim 128 = 64 interleaved RoPE
 * pairs (2j, 2j+1), theta_j = base^(-2j/128), and a group of g consecutive scalars
 * sharing one index per round (review page, "key_machinery"):
 *   g = 8  (default): key 16 groups of 4 pairs, value 16 groups of 8 dims, 256
 *          codewords per (group, round), R = 1 or 2 -> 1 or 2 bits per scalar;
 *          codes token-major [B, Hkv, t_cap, R, 16];
 *   g = 64 (the paper's own parameterization; CommVQ summary page, "Key results" and
 *          "Limitations"): key 2 groups of 32 pairs, value 2 groups of 64 dims, 64
 *          codewords per (group, round), R = 1..22 (11 -> 1.03 bits, 21 -> 1.97 bits
 *          per scalar; each 6-bit code is stored in one uint8);
 *          codes planar [B, Hkv, 2, R, t_cap], t_cap a multiple of 16, one byte per
 *          code; or, with code_bits = 6, packed 4 codes in 3 bytes along each row
 *          (planar [B, Hkv, 2, R, 3 t_cap / 4] bytes, t_cap a multiple of 64), which
 *          stores exactly R x 6 / 64 bits per scalar.
 *   score_t = sum_j Re(e^{i theta_j t} conj(q_j) sum_r c_{t,r,j}) / sqrt(128), t = 0..L-1
 *   out = sum_t softmax(score)_t v_t,   lse = ln sum_t exp(score_t).
 * Query head hq reads KV head hq / (n_q_heads / n_kv_heads).
 * Every entry point takes g = 8; all but cvq_qtable and cvq_decode_attn (the table
 * form) also take g = 64 (the GQA decode with 4 query heads per KV head), and those two
 * return CVQ_ERR_UNSUPPORTED for it.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers, owned by the caller, row-major, and
 *     16-byte aligned.  The library allocates nothing; the only state it keeps between
 *     calls is one device fault word per GPU (cvq_fault_status).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t, NULL = legacy
 *     default stream).  A status of CVQ_OK means the launch was accepted.
 *   - Argument errors are detected on the host before any launch and returned as a
 *     status; nothing is launched then.  Launch failures map to CVQ_ERR_CUDA.  No call
 *     throws across the ABI.
 *   - seq_lens[b] is read on the device and clamped to [0, t_cap].
 *   - The first GQA decode call on a device (cvq_decode_attn_gqa, cvq_attend,
 *     cvq_attend_static) looks up the device fault word's address with that device
 *     current; make it before any stream capture.
 *   - Per device, the library remembers the device addresses of its own device variables
 *     (fault word, static scratch) and the shared-memory limit it set on each kernel.  Like
 *     any state tied to a CUDA context, these do not survive cudaDeviceReset: do not call
 *     the library on a device after resetting it in the same process.
 */
#ifndef CVQ_H
#define CVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CVQ_API __attribute__((visibility("default")))
#else
#define CVQ_API
#endif

#define CVQ_ABI_VERSION 3
#define CVQ_HEAD_DIM 128
#define CVQ_GROUPS 16
#define CVQ_CODES 256

typedef enum {
  CVQ_OK = 0,
  CVQ_ERR_NULL = 1,        /* a required pointer is NULL                            */
  CVQ_ERR_SHAPE = 2,       /* inconsistent or out-of-range sizes                    */
  CVQ_ERR_ALIGN = 3,       /* a pointer (or a codebook head stride) is not 16-byte aligned */
  CVQ_ERR_UNSUPPORTED = 4, /* valid but not implemented (head_dim != 128, R > 2 ...) */
  CVQ_ERR_WORKSPACE = 5,   /* n_splits out of range                                 */
  CVQ_ERR_CUDA = 6,        /* the CUDA runtime reported an error                    */
  CVQ_ERR_STATIC_LIMIT = 7 /* cvq_attend_static: partials exceed the static scratch  */
} cvq_status;

typedef enum { CVQ_F32 = 0, CVQ_BF16 = 1 } cvq_dtype;

typedef struct {
  int32_t batch;      /* 1 <= B <= 65535                                      */
  int32_t n_q_heads;  /* 1 <= Hq <= 65535, a multiple of n_kv_heads          */
  int32_t n_kv_heads; /* Hkv >= 1; Hq/Hkv in {1, 2, 4, 8}                     */
  int32_t head_dim;   /* must be 128                                          */
  int32_t R;          /* residual rounds: 1 or 2 (g = 8), 1..22 (g = 64)      */
  int32_t t_cap;      /* token capacity of the code buffers per sequence, >= 0
                         (group_dim 64: a multiple of 16)                      */
  float rope_base;    /* RoPE base, > 1 (500000 for LLaMA-3.1)                */
  int32_t group_dim;  /* scalars per quantization group: 0 or 8 (default), 64 */
  int32_t code_bits;  /* storage of a code: 0 or 8 = one byte per code (default);
                         6 = packed, 4 codes in 3 bytes (group_dim 64 only, t_cap a
                         multiple of 64; see cvq_pack_codes6)                   */
} cvq_shape;

/* Human-readable name of a status code (static storage). */
CVQ_API const char* cvq_status_str(int status);

/* CVQ_ABI_VERSION of the loaded library. */
CVQ_API int cvq_abi_version(void);

/* ---------------------------------------------------------------------------------
 * cvq_qtable -- the query x key-codebook table, built once per query.
 *   (review page "key_machinery": query-dependent and codebook-dependent factors are
 *    computed once and reused across all cached positions)
 *
 *   P[b, hq, G, r, c, p, 0:2] = conj(q_j) * c,  j = 4G + p,
 *   q_j = q[b, hq, 2j] + i q[b, hq, 2j+1],  c = key_cb[h][G, r, c, p, 0] + i ...[1],
 *   h = hq / (Hq / Hkv).  Unscaled (no 1/sqrt(128)).
 *
 *   q        [B, Hq, 128]           fp32 or bf16 (q_dtype), the already-rotated query
 *   key_cb   [Hkv][16, R, 256, 4, 2] fp32; KV head h starts at key_cb + h * key_cb_head_stride
 *            (stride in floats; 0 = one codebook shared by all KV heads, otherwise
 *            >= 16*R*256*8; a multiple of 4 so every head starts 16-byte aligned, else
 *            CVQ_ERR_ALIGN)
 *   ptable   [B, Hq, 16, R, 256, 4, 2] fp32 output, cvq_ptable_bytes(shape) bytes
 * ------------------------------------------------------------------------------- */
CVQ_API size_t cvq_ptable_bytes(const cvq_shape* shape);
CVQ_API cvq_status cvq_qtable(const cvq_shape* shape, const void* q, int q_dtype, const float* key_cb,
                      int64_t key_cb_head_stride, float* ptable, void* stream);

/* ---------------------------------------------------------------------------------
 * Split-T partial states.  Split s of sequence b covers tokens
 *   [s*C, min((s+1)*C, seq_len[b])),  C = cvq_split_tokens(shape, n_splits)
 * (C is ceil(t_cap / n_splits) rounded up to a multiple of 64), so a split may be
 * empty; an empty split stores m = -inf, l = 0, o = 0.
 *   part_o [B, Hq, n_splits, 128]  sum_t e^{s_t - m} v_t   (unnormalized)
 *   part_m [B, Hq, n_splits]       reference m, natural-log units, with
 *                                  max_t s_t - 8 ln 2 <= m <= max_t s_t
 *   part_l [B, Hq, n_splits]       l = sum_t e^{s_t - m}
 * (m may lag the split maximum by up to 8 ln 2 so that the decode rescales its
 * accumulators rarely; m + ln l and o / l do not depend on it.)
 * cvq_partials_bytes() is the total of the three arrays; 1 <= n_splits <= 4096.
 * ------------------------------------------------------------------------------- */
CVQ_API size_t cvq_partials_bytes(const cvq_shape* shape, int n_splits);
CVQ_API int32_t cvq_split_tokens(const cvq_shape* shape, int n_splits);
/* A split count for this shape on `sm_count` SMs (a suggestion): the count that minimizes
   waves x (split length + a fixed per-CTA cost), the fewest on a tie. */
CVQ_API int cvq_suggest_splits(const cvq_shape* shape, int sm_count);

/* ---------------------------------------------------------------------------------
 * cvq_decode_attn -- split-T flash-decode over the code stream, table form.
 *   (CommVQ summary page "Approach"; review page "key_machinery" and
 *    "forward_implications" 4th item)
 *   For each (b, hq, split): gather sum_r P[G, r, key_code, p] per pair, multiply by
 *   the RoPE phase e^{i theta_j t}, take the real part and sum over pairs -> score;
 *   online softmax; accumulate the weights per value code (bins[G, r, c]); finally
 *   o = bins x val_cb.
 *
 *   ptable     output of cvq_qtable for the same shape
 *   key_codes  [B, Hkv, t_cap, R, 16] uint8  (16-byte aligned)
 *   val_codes  [B, Hkv, t_cap, R, 16] uint8
 *   seq_lens   [B] int32 (device)
 *   val_cb     [Hkv][16, R, 256, 8] fp32, KV head h at val_cb + h * val_cb_head_stride
 *              (0 = shared, otherwise >= 16*R*256*8 and a multiple of 4)
 *   part_*     split partial states, see above
 * ------------------------------------------------------------------------------- */
CVQ_API cvq_status cvq_decode_attn(const cvq_shape* shape, const float* ptable, const uint8_t* key_codes,
                           const uint8_t* val_codes, const int32_t* seq_lens, const float* val_cb,
                           int64_t val_cb_head_stride, int n_splits, float* part_o, float* part_m,
                           float* part_l, void* stream);

/* ---------------------------------------------------------------------------------
 * cvq_decode_attn_gqa -- the same partial states, computed per KV head for all of its
 * Hq/Hkv query heads at once: each token's key codewords are gathered and rotated by
 * the RoPE phase once (the codebook commutes with the rotation, so rotating the
 * codeword equals rotating the key) and projected on every query head of the group.
 *   Same score as cvq_decode_attn up to rounding:
 *     Re(e^{i theta t} conj(q) c) = Re(conj(q) (e^{i theta t} c)).
 *   q, q_dtype, key_cb, key_cb_head_stride as in cvq_qtable; the rest as in
 *   cvq_decode_attn.
 *   With group_dim = 64 (Hq / Hkv must be 4):
 *     key_cb     [Hkv][2, R, 64, 32, 2] fp32 (group G, round r, code c, pair p, re/im;
 *                pair j = 32 G + p), stride 0 or >= 2*R*64*64 floats
 *     val_cb     [Hkv][2, R, 64, 64] fp32 (value dim 64 G + d), same stride rule
 *     key_codes, val_codes  planar [B, Hkv, 2, R, t_cap] uint8 (the low 6 bits of
 *                each byte are the code; the top 2 bits are ignored), t_cap a multiple
 *                of 16 (else CVQ_ERR_SHAPE); with code_bits = 6 packed planar
 *                [B, Hkv, 2, R, 3 t_cap / 4] bytes (layout at cvq_pack_codes6), t_cap a
 *                multiple of 64 (else CVQ_ERR_SHAPE)
 * ------------------------------------------------------------------------------- */
CVQ_API cvq_status cvq_decode_attn_gqa(const cvq_shape* shape, const void* q, int q_dtype,
                               const float* key_cb, int64_t key_cb_head_stride,
                               const uint8_t* key_codes, const uint8_t* val_codes,
                               const int32_t* seq_lens, const float* val_cb,
                               int64_t val_cb_head_stride, int n_splits, float* part_o,
                               float* part_m, float* part_l, void* stream);

/* ---------------------------------------------------------------------------------
 * cvq_attend -- one decode step in one launch: cvq_decode_attn_gqa with the merge of
 * cvq_combine fused into its end.  Each CTA of a work unit (sequence, KV head) counts
 * itself in after writing its partial states; the CTA that arrives last merges the
 * unit's query heads into out and lse (the arithmetic of cvq_combine, in the same order,
 * so the results equal decode + combine bit for bit) and resets the unit's counter.  No
 * CTA waits for another.
 *
 *   Inputs as in cvq_decode_attn_gqa (both group sizes); out [B, Hq, 128] and lse
 *   [B, Hq] as in cvq_combine.
 *   workspace  cvq_attend_workspace_bytes(shape, n_splits) bytes of device memory,
 *              16-byte aligned, owned by the caller: the split partial states followed
 *              by one int32 arrival counter per (sequence, head).  The counters sit
 *              right after the partial states, so their offset depends on the shape
 *              and n_splits.  They must be zero when a call starts: clear the
 *              workspace after allocating it.  A call that completes leaves its own
 *              counters zero, so later calls with the SAME shape and n_splits need no
 *              clearing; before reusing a workspace with a different shape or n_splits,
 *              clear it again (its counters would otherwise land on earlier partial
 *              states).  Calls that share a workspace must be ordered on one stream.
 * ------------------------------------------------------------------------------- */
CVQ_API size_t cvq_attend_workspace_bytes(const cvq_shape* shape, int n_splits);
CVQ_API cvq_status cvq_attend(const cvq_shape* shape, const void* q, int q_dtype,
                              const float* key_cb, int64_t key_cb_head_stride,
                              const uint8_t* key_codes, const uint8_t* val_codes,
                              const int32_t* seq_lens, const float* val_cb,
                              int64_t val_cb_head_stride, int n_splits, void* workspace,
                              float* out, float* lse, void* stream);

/* ---------------------------------------------------------------------------------
 * cvq_combine -- merge split partial states (log-sum-exp):
 *   M = max_s m_s;  L = sum_s l_s e^{m_s - M};
 *   out[b, hq, :] = sum_s o_s e^{m_s - M} / L;   lse[b, hq] = M + ln L.
 *   All splits empty (seq_len 0): out = 0, lse = -inf.
 *   out [B, Hq, 128] fp32, lse [B, Hq] fp32.
 * ------------------------------------------------------------------------------- */
CVQ_API cvq_status cvq_combine(const cvq_shape* shape, int n_splits, const float* part_o,
                       const float* part_m, const float* part_l, float* out, float* lse,
                       void* stream);

/* ---------------------------------------------------------------------------------
 * The naive path, for comparison (CommVQ summary page, "Key results": the optimized
 * commutative-codebook implementation is measured against a naive implementation that
 * decodes the cache before attending).  Not used by the calls above.
 *
 * cvq_naive_dequant -- decode every cached token into fp16 in HBM:
 *   k_out[b, h, t, :] = RoPE_t(sum_r key codewords)  (keys rotated by position t),
 *   v_out[b, h, t, :] = sum_r value codewords,       for t < seq_len[b];
 *   k_out, v_out: [B, Hkv, t_cap, 128] fp16 (IEEE half bits), cvq_naive_cache_bytes() each;
 *   entries t >= seq_len[b] are left untouched.  Other arguments as in cvq_decode_attn_gqa.
 * cvq_naive_decode -- ordinary split-T decode attention over those fp16 keys and values
 *   for every query head (Hq/Hkv <= 4); the same partial states as cvq_decode_attn (here m
 *   is the exact split maximum); merge them with cvq_combine.
 * ------------------------------------------------------------------------------- */
CVQ_API size_t cvq_naive_cache_bytes(const cvq_shape* shape);
CVQ_API cvq_status cvq_naive_dequant(const cvq_shape* shape, const float* key_cb,
                                     int64_t key_cb_head_stride, const uint8_t* key_codes,
                                     const uint8_t* val_codes, const int32_t* seq_lens,
                                     const float* val_cb, int64_t val_cb_head_stride, void* k_out,
                                     void* v_out, void* stream);
CVQ_API cvq_status cvq_naive_decode(const cvq_shape* shape, const void* q, int q_dtype,
                                    const void* k, const void* v, const int32_t* seq_lens,
                                    int n_splits, float* part_o, float* part_m, float* part_l,
                                    void* stream);

/* ---------------------------------------------------------------------------------
 * cvq_encode_append -- the write side of a decode step: quantize one new key and one
 * new value per (sequence, KV head) and store their codes at position positions[b] of
 * the code cache.  The pages encode with a learned encoder (CommVQ abstract; summary
 * page "Approach"), which needs trained weights; this call is the plain stand-in,
 * greedy additive quantization (review page, "key_machinery": R residual rounds refine
 * the reconstruction): for each group G and round r = 0..R-1 it picks the codeword
 * nearest to the running residual and subtracts it.  The squared distance is summed
 * in fp32 over the 8 dims in order 0..7 with no fused multiply-add; ties go to the
 * smaller code.  Keys are encoded before RoPE (the cache holds pre-RoPE keys).
 *
 *   keys, values  [B, Hkv, 128] fp32 (16-byte aligned); a key group G is its pairs
 *                 4G..4G+3 as dims 8G..8G+7 (re, im interleaved), a value group G is
 *                 dims 8G..8G+7 (with group_dim = 64: pairs 32G..32G+31 and dims
 *                 64G..64G+63, 64 codewords per (group, round), distances summed over
 *                 the 64 dims in order)
 *   key_cb, val_cb and their head strides as in cvq_decode_attn_gqa
 *   positions     [B] int32 (device): the token index t each sequence writes; an index
 *                 outside [0, t_cap) writes nothing for that sequence
 *   key_codes, val_codes  [B, Hkv, t_cap, R, 16] uint8, written at [b, h, positions[b]]
 *                 (group_dim = 64: planar [B, Hkv, 2, R, t_cap], written at
 *                 [b, h, :, :, positions[b]]; with code_bits = 6 the packed planar rows,
 *                 where only the 6 bits of code positions[b] change in each row) and
 *                 nowhere else (the caller owns them; seq_lens is the caller's to
 *                 advance).  Calls that write the same rows must be ordered on one
 *                 stream (a packed code shares its bytes with its neighbours).
 *   Errors: CVQ_ERR_NULL / CVQ_ERR_ALIGN / CVQ_ERR_SHAPE / CVQ_ERR_UNSUPPORTED before any
 *   launch; CVQ_ERR_CUDA if the launch fails.  Asynchronous on `stream`.
 * ------------------------------------------------------------------------------- */
CVQ_API cvq_status cvq_encode_append(const cvq_shape* shape, const float* keys, const float* values,
                                     const float* key_cb, int64_t key_cb_head_stride,
                                     const float* val_cb, int64_t val_cb_head_stride,
                                     const int32_t* positions, uint8_t* key_codes,
                                     uint8_t* val_codes, void* stream);

/* ---------------------------------------------------------------------------------
 * cvq_pack_codes6 -- repack the paper's 6-bit codes from one byte per code to 4 codes in
 * 3 bytes (CommVQ summary page, "Key results": 64-entry codebooks, so R = 11 rounds
 * over 64-scalar groups store 11 x 6 / 64 = 1.03 bits per scalar).  The pages fix no bit
 * layout; this one is little-endian along each row of the planar layout: codes
 * t = 4i .. 4i+3 of a (sequence, KV head, group, round) row form the 24-bit
 * little-endian word in bytes 3i .. 3i+2, code 4i + j in bits 6j .. 6j+5.
 *   shape      group_dim 64, code_bits 6 (the layout being produced), t_cap a multiple
 *              of 64
 *   codes_in   planar [B, Hkv, 2, R, t_cap] uint8, one code per byte (low 6 bits used),
 *              16-byte aligned
 *   packed_out planar [B, Hkv, 2, R, 3 t_cap / 4] uint8, 16-byte aligned; every byte
 *              is written (every token up to t_cap, whatever the sequence lengths)
 *   Errors: CVQ_ERR_NULL / CVQ_ERR_ALIGN / CVQ_ERR_SHAPE / CVQ_ERR_UNSUPPORTED before any
 *   launch; CVQ_ERR_CUDA if the launch fails.  Asynchronous on `stream`.
 * ------------------------------------------------------------------------------- */
CVQ_API cvq_status cvq_pack_codes6(const cvq_shape* shape, const uint8_t* codes_in,
                                   uint8_t* packed_out, void* stream);

/* ---------------------------------------------------------------------------------
 * cvq_attend_static -- cvq_attend (decode with the fused split merge, one launch) with
 * its workspace -- the split partial states and the arrival counters -- kept in a fixed
 * device array inside the library instead of memory the caller allocates.  The paper has no counterpart: this is an interface for
 * callers that cannot allocate device memory while decoding -- a serving process
 * whose pool has already claimed all free HBM for the KV cache, a plugin whose host
 * gives it no allocator, or a decode loop that cannot afford cudaMalloc's implicit
 * synchronization.  The call itself allocates nothing.
 *
 *   Arguments as in cvq_decode_attn_gqa, then out [B, Hq, 128] and lse [B, Hq] as in
 *   cvq_combine.  The array (CVQ_STATIC_SCRATCH_BYTES = 4 MiB, held by every GPU that
 *   loads the library until the process exits) has a fixed layout: its first
 *   CVQ_STATIC_COUNTER_BYTES (32 KiB) hold the arrival counters, one int32 per
 *   (sequence, query head), and the rest holds the split partial states.  So a call
 *   fits when cvq_partials_bytes(shape, n_splits) <= 4 MiB - 32 KiB and
 *   batch * n_q_heads <= 8192; any other call returns CVQ_ERR_STATIC_LIMIT before any
 *   launch.  Every call first clears its counters (an asynchronous cudaMemsetAsync on
 *   `stream`, issued after all argument checks; it allocates nothing), so calls of any
 *   shape may follow one another in any order.
 *   The first call on a device looks up the array's device address with that device
 *   current (cudaGetSymbolAddress), so make that first call before any stream capture.
 *   Every call reuses the same array: calls whose work overlaps on the GPU (other
 *   streams, other host threads) race on it and must be serialized by the caller.
 * ------------------------------------------------------------------------------- */
#define CVQ_STATIC_SCRATCH_BYTES (4u * 1024u * 1024u)
#define CVQ_STATIC_COUNTER_BYTES (32u * 1024u)
CVQ_API cvq_status cvq_attend_static(const cvq_shape* shape, const void* q, int q_dtype,
                                     const float* key_cb, int64_t key_cb_head_stride,
                                     const uint8_t* key_codes, const uint8_t* val_codes,
                                     const int32_t* seq_lens, const float* val_cb,
                                     int64_t val_cb_head_stride, int n_splits, float* out,
                                     float* lse, void* stream);

/* ---------------------------------------------------------------------------------
 * cvq_fault_status -- the device fault word of the current device.  The decode kernels
 * that stage codebooks with the TMA engine (cvq_decode_attn_gqa / cvq_attend /
 * cvq_attend_static with 4 query heads per KV head, and every g = 64 decode) wait for
 * those copies with a bounded wait; if a wait gives up, the kernel sets a bit here and
 * runs to completion (its outputs are then invalid) instead of hanging the GPU.
 *   Bits: CVQ_FAULT_COPY_TIMEOUT = a codebook copy (or, in a decode kernel, a wait on a
 *         shared-memory barrier) did not complete within the wait limit;
 *         CVQ_FAULT_BOUNDS = a device-side range check failed.  Only the debug build of
 *         the library (compiled with -DCVQ_DEBUG_BOUNDS, libcvq_debug.so) has these checks:
 *         the code row of every code copy, every codeword and bin index, the exchange index
 *         between the CTAs of a pair, and the partial-state rows and arrival counter of
 *         every work unit.  A failed check skips its access (a skipped load reads 0) and
 *         the kernel runs on; the outputs of that call are then invalid.
 *   flags (host): receives the word.  clear != 0 resets it to 0 afterwards.
 *   Synchronous: waits for the device (cudaMemcpy).  The first call on a device looks up
 *   the word's address (cudaGetSymbolAddress), as the first decode call does; make that
 *   first call before any stream capture.
 *   Errors: CVQ_ERR_NULL (flags NULL), CVQ_ERR_CUDA.
 * ------------------------------------------------------------------------------- */
#define CVQ_FAULT_COPY_TIMEOUT 1u
#define CVQ_FAULT_BOUNDS 2u
CVQ_API cvq_status cvq_fault_status(uint32_t* flags, int clear);

#ifdef __cplusplus
}
#endif
#endif /* CVQ_H */
