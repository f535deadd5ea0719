// libcvq C ABI: argument validation on the host, then kernel launches.  Nothing is
// allocated; the only state is the device fault word (device_state.cu).  Every argument
// error is returned as a cvq_status before any launch.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "common.cuh"

using namespace cvq;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_wide(const cvq_shape* s) { return s->group_dim == kWideGroupDim; }

// floats of one KV head's key / value codebook
size_t key_cb_floats(const cvq_shape* s) {
  return is_wide(s) ? static_cast<size_t>(kWideGroups) * s->R * kWideCodes * 2 * kWidePairs
                    : static_cast<size_t>(kGroups) * s->R * kCodes * kCodeword;
}
size_t val_cb_floats(const cvq_shape* s) {
  return is_wide(s) ? static_cast<size_t>(kWideGroups) * s->R * kWideCodes * kWideVDims
                    : static_cast<size_t>(kGroups) * s->R * kCodes * kVDims;
}

cvq_status check_shape(const cvq_shape* s) {
  if (s == nullptr) return CVQ_ERR_NULL;
  if (s->head_dim != kHeadDim) return CVQ_ERR_UNSUPPORTED;
  if (s->group_dim != 0 && s->group_dim != 8 && s->group_dim != kWideGroupDim)
    return CVQ_ERR_UNSUPPORTED;
  if (s->code_bits != 0 && s->code_bits != 8 && s->code_bits != 6) return CVQ_ERR_UNSUPPORTED;
  if (is_wide(s)) {
    if (s->R < 1 || s->R > kWideMaxR) return CVQ_ERR_UNSUPPORTED;
    if (s->t_cap % 16 != 0) return CVQ_ERR_SHAPE;      // planar code rows in 16-byte chunks
    // packed rows: 64 codes = 48 bytes, so every row and every 64-token chunk of it
    // starts on a 16-byte boundary
    if (s->code_bits == 6 && s->t_cap % 64 != 0) return CVQ_ERR_SHAPE;
  } else if (s->R != 1 && s->R != 2) {
    return CVQ_ERR_UNSUPPORTED;
  } else if (s->code_bits == 6) {
    return CVQ_ERR_UNSUPPORTED;                        // 6-bit codes: 64-entry codebooks only
  }
  if (s->batch < 1 || s->n_q_heads < 1 || s->n_kv_heads < 1 || s->t_cap < 0) return CVQ_ERR_SHAPE;
  if (s->n_q_heads % s->n_kv_heads != 0) return CVQ_ERR_SHAPE;
  if (s->batch > 65535 || s->n_q_heads > 65535) return CVQ_ERR_SHAPE;
  if (!std::isfinite(s->rope_base) || !(s->rope_base > 1.0f)) return CVQ_ERR_SHAPE;
  const int g = s->n_q_heads / s->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return CVQ_ERR_UNSUPPORTED;
  return CVQ_OK;
}

cvq_status check_stride(int64_t stride, size_t per_head) {
  if (stride < 0) return CVQ_ERR_SHAPE;
  if (stride != 0 && static_cast<uint64_t>(stride) < per_head) return CVQ_ERR_SHAPE;
  if (stride % 4 != 0) return CVQ_ERR_ALIGN;   // every head's codebook 16-byte aligned
  return CVQ_OK;
}

cvq_status check_ptr(const void* p) {
  if (p == nullptr) return CVQ_ERR_NULL;
  if (!aligned16(p)) return CVQ_ERR_ALIGN;
  return CVQ_OK;
}

#define CVQ_TRY(expr)                 \
  do {                                \
    const cvq_status st_ = (expr);    \
    if (st_ != CVQ_OK) return st_;    \
  } while (0)

cvq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CVQ_OK : CVQ_ERR_CUDA; }

cvq_status check_decode_common(const cvq_shape* s, const uint8_t* key_codes, const uint8_t* val_codes,
                               const int32_t* seq_lens, const float* val_cb, int64_t val_stride,
                               int n_splits, float* part_o, float* part_m, float* part_l) {
  CVQ_TRY(check_ptr(key_codes));
  CVQ_TRY(check_ptr(val_codes));
  if (seq_lens == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(seq_lens) & 3u) != 0) return CVQ_ERR_ALIGN;
  CVQ_TRY(check_ptr(val_cb));
  CVQ_TRY(check_stride(val_stride, val_cb_floats(s)));
  if (n_splits < 1 || n_splits > 4096) return CVQ_ERR_WORKSPACE;
  CVQ_TRY(check_ptr(part_o));
  if (part_m == nullptr || part_l == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(part_m) & 3u) || (reinterpret_cast<uintptr_t>(part_l) & 3u))
    return CVQ_ERR_ALIGN;
  return CVQ_OK;
}

void fill_common(DecodeArgs& a, const cvq_shape* s, const uint8_t* key_codes, const uint8_t* val_codes,
                 const int32_t* seq_lens, const float* val_cb, int64_t val_stride, int n_splits,
                 float* part_o, float* part_m, float* part_l) {
  a.key_codes = key_codes;
  a.val_codes = val_codes;
  a.seq_lens = seq_lens;
  a.val_cb = val_cb;
  a.val_cb_stride = val_stride;
  a.batch = s->batch;
  a.n_q_heads = s->n_q_heads;
  a.n_kv_heads = s->n_kv_heads;
  a.t_cap = s->t_cap;
  a.code_bits = s->code_bits == 6 ? 6 : 8;
  a.n_splits = n_splits;
  a.split_tokens = split_tokens_host(s->t_cap, n_splits);
  a.part_o = part_o;
  a.part_m = part_m;
  a.part_l = part_l;
  phase_turns_host(s->rope_base, &a.phase);
}

size_t round16(size_t n) { return (n + 15) / 16 * 16; }

// The GQA-form decode; with counters != nullptr the last CTA of every work unit also merges
// the split partials into out and lse (cvq_attend).
cvq_status decode_gqa_impl(const cvq_shape* s, const void* q, int q_dtype, const float* key_cb,
                           int64_t key_cb_head_stride, const uint8_t* key_codes,
                           const uint8_t* val_codes, const int32_t* seq_lens, const float* val_cb,
                           int64_t val_cb_head_stride, int n_splits, float* part_o, float* part_m,
                           float* part_l, int* counters, float* out, float* lse, void* stream,
                           size_t clear_counters = 0) {
  CVQ_TRY(check_shape(s));
  if (q_dtype != CVQ_F32 && q_dtype != CVQ_BF16) return CVQ_ERR_UNSUPPORTED;
  CVQ_TRY(check_ptr(q));
  CVQ_TRY(check_ptr(key_cb));
  CVQ_TRY(check_stride(key_cb_head_stride, key_cb_floats(s)));
  if (is_wide(s) ? (s->n_q_heads / s->n_kv_heads) != 4
                 : (s->n_q_heads / s->n_kv_heads) * s->R > 8)
    return CVQ_ERR_UNSUPPORTED;
  CVQ_TRY(check_decode_common(s, key_codes, val_codes, seq_lens, val_cb, val_cb_head_stride,
                              n_splits, part_o, part_m, part_l));
  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  fill_common(a, s, key_codes, val_codes, seq_lens, val_cb, val_cb_head_stride, n_splits, part_o,
              part_m, part_l);
  a.key_tab = key_cb;
  a.key_tab_stride = key_cb_head_stride;
  a.q = q;
  a.q_dtype = q_dtype;
  a.counters = counters;
  a.out = out;
  a.lse = lse;
  if (fault_word_address(&a.fault) != cudaSuccess) return CVQ_ERR_CUDA;
  if (!is_wide(s) && s->n_q_heads / s->n_kv_heads == 4) {   // the kernel that stages by TMA maps
    if (encode_codebook_map(&a.key_map, key_cb, key_cb_head_stride, s->n_kv_heads, s->R) != cudaSuccess ||
        encode_codebook_map(&a.val_map, val_cb, val_cb_head_stride, s->n_kv_heads, s->R) != cudaSuccess)
      return CVQ_ERR_CUDA;
  }
  // every argument is valid: clear the counters first if the caller asked (enqueued on the
  // same stream, so the decode kernel sees them zero)
  if (clear_counters != 0 &&
      cudaMemsetAsync(counters, 0, clear_counters * sizeof(int), static_cast<cudaStream_t>(stream)) !=
          cudaSuccess)
    return CVQ_ERR_CUDA;
  if (is_wide(s)) return from_cuda(launch_decode_wide(*s, a, static_cast<cudaStream_t>(stream)));
  return from_cuda(launch_decode_gqa(*s, a, static_cast<cudaStream_t>(stream)));
}

}  // namespace

namespace cvq {

// F_j for every pair, computed in long double
static void phase_turns_exact(float rope_base, PhaseTurns* out) {
  const long double two_pi = 6.283185307179586476925286766559L;
  const long double base = static_cast<long double>(rope_base);
  for (int j = 0; j < kPairs; ++j) {
    const long double theta = powl(base, -2.0L * j / kHeadDim);
    long double turns = theta / two_pi;                  // < 1 turn per token
    turns -= floorl(turns);
    const long double scaled = ldexpl(turns, 64);        // in [0, 2^64)
    unsigned long long f;
    if (scaled >= 18446744073709551615.0L) {
      f = ~0ULL;
    } else {
      f = static_cast<unsigned long long>(scaled + 0.5L);
    }
    out->F[j] = f;
  }
}

// The turns depend on rope_base alone, and a decode loop passes the same base at every
// step, while the 64 long-double powers cost ~20 us of host time: each calling thread keeps
// the turns of the last base it asked for.
void phase_turns_host(float rope_base, PhaseTurns* out) {
  thread_local bool have = false;
  thread_local uint32_t have_bits = 0;
  thread_local PhaseTurns have_turns;
  uint32_t bits;
  std::memcpy(&bits, &rope_base, sizeof(bits));
  if (!have || bits != have_bits) {
    phase_turns_exact(rope_base, &have_turns);
    have_bits = bits;
    have = true;
  }
  *out = have_turns;
}

cvq_status attend_into(const cvq_shape* s, const void* q, int q_dtype, const float* key_cb,
                       int64_t key_cb_head_stride, const uint8_t* key_codes,
                       const uint8_t* val_codes, const int32_t* seq_lens, const float* val_cb,
                       int64_t val_cb_head_stride, int n_splits, float* partials, int* counters,
                       float* out, float* lse, void* stream, size_t clear_counters) {
  CVQ_TRY(check_shape(s));
  CVQ_TRY(check_ptr(partials));
  if (counters == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(counters) & 3u) != 0) return CVQ_ERR_ALIGN;
  CVQ_TRY(check_ptr(out));
  if (lse == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return CVQ_ERR_ALIGN;
  if (n_splits < 1 || n_splits > 4096) return CVQ_ERR_WORKSPACE;
  // partials: part_o [rows][128], part_m [rows], part_l [rows]
  const size_t rows = static_cast<size_t>(s->batch) * s->n_q_heads * n_splits;
  float* part_o = partials;
  float* part_m = part_o + rows * kHeadDim;
  float* part_l = part_m + rows;
  return decode_gqa_impl(s, q, q_dtype, key_cb, key_cb_head_stride, key_codes, val_codes,
                         seq_lens, val_cb, val_cb_head_stride, n_splits, part_o, part_m, part_l,
                         counters, out, lse, stream, clear_counters);
}

}  // namespace cvq

extern "C" {

const char* cvq_status_str(int status) {
  switch (status) {
    case CVQ_OK: return "CVQ_OK";
    case CVQ_ERR_NULL: return "CVQ_ERR_NULL: a required pointer is NULL";
    case CVQ_ERR_SHAPE: return "CVQ_ERR_SHAPE: inconsistent or out-of-range sizes";
    case CVQ_ERR_ALIGN: return "CVQ_ERR_ALIGN: a pointer is not 16-byte aligned";
    case CVQ_ERR_UNSUPPORTED: return "CVQ_ERR_UNSUPPORTED: head_dim, R, dtype or GQA group not supported";
    case CVQ_ERR_WORKSPACE: return "CVQ_ERR_WORKSPACE: n_splits out of range";
    case CVQ_ERR_CUDA: return "CVQ_ERR_CUDA: the CUDA runtime reported an error";
    case CVQ_ERR_STATIC_LIMIT: return "CVQ_ERR_STATIC_LIMIT: the partial states exceed the static scratch";
    default: return "unknown cvq_status";
  }
}

int cvq_abi_version(void) { return CVQ_ABI_VERSION; }

size_t cvq_ptable_bytes(const cvq_shape* s) {
  if (check_shape(s) != CVQ_OK || is_wide(s)) return 0;
  return static_cast<size_t>(s->batch) * s->n_q_heads * key_cb_floats(s) * sizeof(float);
}

size_t cvq_partials_bytes(const cvq_shape* s, int n_splits) {
  if (check_shape(s) != CVQ_OK || n_splits < 1 || n_splits > 4096) return 0;
  const size_t rows = static_cast<size_t>(s->batch) * s->n_q_heads * n_splits;
  return rows * (kHeadDim + 2) * sizeof(float);
}

int32_t cvq_split_tokens(const cvq_shape* s, int n_splits) {
  if (check_shape(s) != CVQ_OK || n_splits < 1 || n_splits > 4096) return 0;
  return split_tokens_host(s->t_cap, n_splits);
}

int cvq_suggest_splits(const cvq_shape* s, int sm_count) {
  if (check_shape(s) != CVQ_OK || sm_count < 1) return 1;
  // CTAs per split index and CTA slots on the GPU: the 4-head kernel runs a cluster of 2
  // CTAs per (sequence, KV head, split), 2 per SM at R = 1 and 1 per SM at R = 2; with
  // 64-scalar groups a cluster of 2 * ceil(R / 11) CTAs, one per SM; the plain kernel runs
  // one CTA per (sequence, KV head, split).  Every split of a launch is equally long, so a
  // launch takes about waves x (split length + a fixed cost per CTA for loading the
  // codebooks and the epilogue, ~min_len tokens' worth); take the split count that
  // minimizes that, the fewest splits on a tie.
  const bool clustered = (s->n_q_heads / s->n_kv_heads) == 4;
  const long long per_split = is_wide(s) ? wide_cluster_size(s->R) : (clustered ? 2 : 1);
  const long long units = static_cast<long long>(s->batch) * s->n_kv_heads * per_split;
  const long long slots =
      static_cast<long long>(sm_count) * (clustered && !is_wide(s) && s->R == 1 ? 2 : 1);
  const long long min_len = clustered ? 256LL : 64LL;
  const long long max_splits = std::max(1LL, std::min(4096LL, (s->t_cap + min_len - 1) / min_len));
  long long best_n = 1, best_cost = -1;
  for (long long n = 1; n <= max_splits; ++n) {
    const long long waves = (units * n + slots - 1) / slots;
    const long long len = split_tokens_host(s->t_cap, static_cast<int>(n));
    const long long cost = waves * (len + min_len);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_n = n;
    }
  }
  return static_cast<int>(best_n);
}

cvq_status cvq_qtable(const cvq_shape* s, const void* q, int q_dtype, const float* key_cb,
                      int64_t key_cb_head_stride, float* ptable, void* stream) {
  CVQ_TRY(check_shape(s));
  if (is_wide(s)) return CVQ_ERR_UNSUPPORTED;
  if (q_dtype != CVQ_F32 && q_dtype != CVQ_BF16) return CVQ_ERR_UNSUPPORTED;
  CVQ_TRY(check_ptr(q));
  CVQ_TRY(check_ptr(key_cb));
  CVQ_TRY(check_ptr(ptable));
  CVQ_TRY(check_stride(key_cb_head_stride, key_cb_floats(s)));
  return from_cuda(launch_qtable(*s, q, q_dtype, key_cb, key_cb_head_stride, ptable,
                                 static_cast<cudaStream_t>(stream)));
}

cvq_status cvq_decode_attn(const cvq_shape* s, const float* ptable, const uint8_t* key_codes,
                           const uint8_t* val_codes, const int32_t* seq_lens, const float* val_cb,
                           int64_t val_cb_head_stride, int n_splits, float* part_o, float* part_m,
                           float* part_l, void* stream) {
  CVQ_TRY(check_shape(s));
  if (is_wide(s)) return CVQ_ERR_UNSUPPORTED;
  CVQ_TRY(check_ptr(ptable));
  CVQ_TRY(check_decode_common(s, key_codes, val_codes, seq_lens, val_cb, val_cb_head_stride,
                              n_splits, part_o, part_m, part_l));
  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  fill_common(a, s, key_codes, val_codes, seq_lens, val_cb, val_cb_head_stride, n_splits, part_o,
              part_m, part_l);
  a.key_tab = ptable;
  a.key_tab_stride = static_cast<long long>(key_cb_floats(s));
  return from_cuda(launch_decode_table(*s, a, static_cast<cudaStream_t>(stream)));
}

cvq_status cvq_decode_attn_gqa(const cvq_shape* s, const void* q, int q_dtype, const float* key_cb,
                               int64_t key_cb_head_stride, const uint8_t* key_codes,
                               const uint8_t* val_codes, const int32_t* seq_lens,
                               const float* val_cb, int64_t val_cb_head_stride, int n_splits,
                               float* part_o, float* part_m, float* part_l, void* stream) {
  return decode_gqa_impl(s, q, q_dtype, key_cb, key_cb_head_stride, key_codes, val_codes,
                         seq_lens, val_cb, val_cb_head_stride, n_splits, part_o, part_m, part_l,
                         nullptr, nullptr, nullptr, stream);
}

size_t cvq_attend_workspace_bytes(const cvq_shape* s, int n_splits) {
  const size_t parts = cvq_partials_bytes(s, n_splits);
  if (parts == 0) return 0;
  return round16(parts) + round16(static_cast<size_t>(s->batch) * s->n_q_heads * sizeof(int));
}

cvq_status cvq_attend(const cvq_shape* s, const void* q, int q_dtype, const float* key_cb,
                      int64_t key_cb_head_stride, const uint8_t* key_codes,
                      const uint8_t* val_codes, const int32_t* seq_lens, const float* val_cb,
                      int64_t val_cb_head_stride, int n_splits, void* workspace, float* out,
                      float* lse, void* stream) {
  CVQ_TRY(check_shape(s));
  CVQ_TRY(check_ptr(workspace));
  CVQ_TRY(check_ptr(out));
  if (lse == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return CVQ_ERR_ALIGN;
  if (n_splits < 1 || n_splits > 4096) return CVQ_ERR_WORKSPACE;
  // workspace: part_o [rows][128], part_m [rows], part_l [rows], then the counters
  const size_t rows = static_cast<size_t>(s->batch) * s->n_q_heads * n_splits;
  int* counters = reinterpret_cast<int*>(static_cast<char*>(workspace) +
                                         round16(rows * (kHeadDim + 2) * sizeof(float)));
  return cvq::attend_into(s, q, q_dtype, key_cb, key_cb_head_stride, key_codes, val_codes,
                          seq_lens, val_cb, val_cb_head_stride, n_splits,
                          static_cast<float*>(workspace), counters, out, lse, stream, 0);
}

cvq_status cvq_combine(const cvq_shape* s, int n_splits, const float* part_o, const float* part_m,
                       const float* part_l, float* out, float* lse, void* stream) {
  CVQ_TRY(check_shape(s));
  if (n_splits < 1 || n_splits > 4096) return CVQ_ERR_WORKSPACE;
  CVQ_TRY(check_ptr(part_o));
  CVQ_TRY(check_ptr(out));
  if (part_m == nullptr || part_l == nullptr || lse == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(part_m) & 3u) || (reinterpret_cast<uintptr_t>(part_l) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return CVQ_ERR_ALIGN;
  return from_cuda(launch_combine(*s, n_splits, part_o, part_m, part_l, out, lse,
                                  static_cast<cudaStream_t>(stream)));
}

size_t cvq_naive_cache_bytes(const cvq_shape* s) {
  if (check_shape(s) != CVQ_OK) return 0;
  return static_cast<size_t>(s->batch) * s->n_kv_heads * s->t_cap * kHeadDim * 2;
}

cvq_status cvq_naive_dequant(const cvq_shape* s, const float* key_cb, int64_t key_cb_head_stride,
                             const uint8_t* key_codes, const uint8_t* val_codes,
                             const int32_t* seq_lens, const float* val_cb,
                             int64_t val_cb_head_stride, void* k_out, void* v_out, void* stream) {
  CVQ_TRY(check_shape(s));
  CVQ_TRY(check_ptr(key_cb));
  CVQ_TRY(check_ptr(val_cb));
  CVQ_TRY(check_ptr(key_codes));
  CVQ_TRY(check_ptr(val_codes));
  CVQ_TRY(check_ptr(k_out));
  CVQ_TRY(check_ptr(v_out));
  if (seq_lens == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(seq_lens) & 3u) != 0) return CVQ_ERR_ALIGN;
  CVQ_TRY(check_stride(key_cb_head_stride, key_cb_floats(s)));
  CVQ_TRY(check_stride(val_cb_head_stride, val_cb_floats(s)));
  PhaseTurns ph;
  phase_turns_host(s->rope_base, &ph);
  return from_cuda(launch_naive_dequant(*s, key_cb, key_cb_head_stride, val_cb, val_cb_head_stride,
                                        key_codes, val_codes, seq_lens, ph, k_out, v_out,
                                        static_cast<cudaStream_t>(stream)));
}

cvq_status cvq_naive_decode(const cvq_shape* s, const void* q, int q_dtype, const void* k,
                            const void* v, const int32_t* seq_lens, int n_splits, float* part_o,
                            float* part_m, float* part_l, void* stream) {
  CVQ_TRY(check_shape(s));
  if (q_dtype != CVQ_F32 && q_dtype != CVQ_BF16) return CVQ_ERR_UNSUPPORTED;
  if (s->n_q_heads / s->n_kv_heads > 4) return CVQ_ERR_UNSUPPORTED;
  CVQ_TRY(check_ptr(q));
  CVQ_TRY(check_ptr(k));
  CVQ_TRY(check_ptr(v));
  if (seq_lens == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(seq_lens) & 3u) != 0) return CVQ_ERR_ALIGN;
  if (n_splits < 1 || n_splits > 4096) return CVQ_ERR_WORKSPACE;
  CVQ_TRY(check_ptr(part_o));
  if (part_m == nullptr || part_l == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(part_m) & 3u) || (reinterpret_cast<uintptr_t>(part_l) & 3u))
    return CVQ_ERR_ALIGN;
  return from_cuda(launch_naive_decode(*s, q, q_dtype, k, v, seq_lens, n_splits,
                                       split_tokens_host(s->t_cap, n_splits), part_o, part_m,
                                       part_l, static_cast<cudaStream_t>(stream)));
}

cvq_status cvq_pack_codes6(const cvq_shape* s, const uint8_t* codes_in, uint8_t* packed_out,
                           void* stream) {
  CVQ_TRY(check_shape(s));
  if (!is_wide(s) || s->code_bits != 6) return CVQ_ERR_UNSUPPORTED;
  CVQ_TRY(check_ptr(codes_in));
  CVQ_TRY(check_ptr(packed_out));
  if (s->t_cap == 0) return CVQ_OK;
  const size_t rows = static_cast<size_t>(s->batch) * s->n_kv_heads * kWideGroups * s->R;
  return from_cuda(launch_pack_codes6(codes_in, packed_out, rows, s->t_cap,
                                      static_cast<cudaStream_t>(stream)));
}

cvq_status cvq_encode_append(const cvq_shape* s, const float* keys, const float* values,
                             const float* key_cb, int64_t key_cb_head_stride, const float* val_cb,
                             int64_t val_cb_head_stride, const int32_t* positions,
                             uint8_t* key_codes, uint8_t* val_codes, void* stream) {
  CVQ_TRY(check_shape(s));
  CVQ_TRY(check_ptr(keys));
  CVQ_TRY(check_ptr(values));
  CVQ_TRY(check_ptr(key_cb));
  CVQ_TRY(check_ptr(val_cb));
  CVQ_TRY(check_ptr(key_codes));
  CVQ_TRY(check_ptr(val_codes));
  if (positions == nullptr) return CVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(positions) & 3u) != 0) return CVQ_ERR_ALIGN;
  CVQ_TRY(check_stride(key_cb_head_stride, key_cb_floats(s)));
  CVQ_TRY(check_stride(val_cb_head_stride, val_cb_floats(s)));
  if (s->t_cap == 0) return CVQ_OK;
  return from_cuda(launch_encode_append(*s, keys, values, key_cb, key_cb_head_stride, val_cb,
                                        val_cb_head_stride, positions, key_codes, val_codes,
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
