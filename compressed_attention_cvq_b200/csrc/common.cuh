// Shared definitions of the libcvq kernels: layout constants, the RoPE phase in exact
// fixed-point turns, and small device helpers.
#pragma once

#include <cuda.h>            // CUtensorMap (the type only; the encoder is reached at run time)
#include <cuda_runtime.h>
#include <atomic>
#include <stdint.h>

#include "cvq.h"

namespace cvq {

constexpr int kHeadDim = 128;
constexpr int kPairs = 64;
constexpr int kGroups = 16;
constexpr int kPairsPerGroup = 4;
constexpr int kVDims = 8;
constexpr int kCodes = 256;
constexpr int kCodeword = 8;              // floats per key codeword (4 pairs x re/im)
constexpr int kSplitAlign = 64;           // split boundaries are multiples of this
// the paper's own parameterization: 64-entry codebooks over groups of 64 scalars
constexpr int kWideGroupDim = 64;
constexpr int kWideGroups = 2;            // groups per head
constexpr int kWidePairs = 32;            // RoPE pairs per key group
constexpr int kWideVDims = 64;            // dims per value group
constexpr int kWideCodes = 64;            // codewords per (group, round)
constexpr int kWideRoundsPerCta = 11;     // rounds one CTA of the cluster holds
constexpr int kWideMaxR = 2 * kWideRoundsPerCta;
// CTAs per (sequence, KV head, split): one per group and round slice of <= 11 rounds
__host__ __device__ constexpr int wide_round_slices(int R) {
  return (R + kWideRoundsPerCta - 1) / kWideRoundsPerCta;
}
__host__ __device__ constexpr int wide_cluster_size(int R) { return kWideGroups * wide_round_slices(R); }
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// RoPE phase of pair j at position t as an exact fraction of a turn:
//   theta_j t / (2 pi) mod 1  ==  (F_j * t mod 2^64) / 2^64,
// with F_j = round(2^64 theta_j / (2 pi)).  The 64-bit wrap-around product performs
// the range reduction exactly, so the angle stays accurate at any position
// (theta_0 t reaches 1.3e5 rad at t = 131072, where an fp32 angle would be off by
// up to ~8e-3 rad).
struct PhaseTurns {
  unsigned long long F[kPairs];
};

// Host: fill F_j for a RoPE base (long double for the 64-bit fraction).
void phase_turns_host(float rope_base, PhaseTurns* out);

// cos/sin of 2 pi * (turn64 / 2^64); the top 32 bits give the angle to 2^-32 turns,
// taken as a signed value so the argument of the sine stays in [-pi, pi).
__device__ __forceinline__ float2 phase_from_turn(unsigned long long turn64) {
  const int hi = static_cast<int>(turn64 >> 32);
  const float ang = static_cast<float>(hi) * 1.4629180792671596e-09f;  // 2 pi / 2^32
  float s, c;
  __sincosf(ang, &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ float2 phase_at(unsigned long long F, int t) {
  return phase_from_turn(F * static_cast<unsigned long long>(static_cast<unsigned>(t)));
}

// Order-preserving map of a float (not NaN) to an int and back, for integer atomicMax.
__device__ __forceinline__ int ord_of(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float float_of_ord(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float load_q(const void* q, int q_dtype, size_t idx) {
  if (q_dtype == CVQ_BF16) return bf16_bits_to_float(static_cast<const uint16_t*>(q)[idx]);
  return static_cast<const float*>(q)[idx];
}

// Code t of a packed row (6 bits per code, 4 codes in 3 bytes, little-endian: code
// 4i + j in bits 6j .. 6j+5 of the 24-bit word in bytes 3i .. 3i+2).  A code lies in one
// byte (j = 0, 3) or two bytes of its own 3-byte group (j = 1, 2); nothing past the
// group is read.
__device__ __forceinline__ int packed6_code(const uint8_t* row, int t) {
  const int bit = 6 * t, by = bit >> 3, sh = bit & 7;
  uint32_t w = row[by];
  if (sh > 2) w |= static_cast<uint32_t>(row[by + 1]) << 8;
  return static_cast<int>((w >> sh) & 63u);
}

__device__ __forceinline__ int code_byte(const uint4& v, int G) {
  const uint32_t w = (G < 4) ? v.x : (G < 8) ? v.y : (G < 12) ? v.z : v.w;
  return static_cast<int>((w >> (8 * (G & 3))) & 0xffu);
}

// First token of split s and the split length (multiple of kSplitAlign).
inline int32_t split_tokens_host(int32_t t_cap, int n_splits) {
  int64_t c = (static_cast<int64_t>(t_cap) + n_splits - 1) / n_splits;
  c = ((c + kSplitAlign - 1) / kSplitAlign) * kSplitAlign;
  if (c < kSplitAlign) c = kSplitAlign;
  return static_cast<int32_t>(c);
}

// Arguments shared by the decode kernels.
struct DecodeArgs {
  const float* key_tab;          // key codebook (per KV head) or P table (per query head)
  long long key_tab_stride;      // floats between consecutive heads of key_tab
  const void* q;                 // queries (GQA form only)
  int q_dtype;
  const uint8_t* key_codes;
  const uint8_t* val_codes;
  const int32_t* seq_lens;
  const float* val_cb;
  long long val_cb_stride;
  int batch, n_q_heads, n_kv_heads, t_cap, n_splits, split_tokens;
  int code_bits;                 // 8: one byte per code; 6: packed (64-scalar groups only)
  float* part_o;
  float* part_m;
  float* part_l;
  PhaseTurns phase;
  // fused merge (cvq_attend): arrival counters per work unit and the final outputs;
  // counters == nullptr leaves the merge to cvq_combine
  int* counters;
  float* out;
  float* lse;
  // 4-query-head kernel only: tiled TMA maps of the key and value codebooks (see
  // encode_codebook_map), read from the kernel parameter space
  CUtensorMap key_map;
  CUtensorMap val_map;
  // device fault word of the library (kFault* bits), set when a bounded wait gives up
  unsigned int* fault;
};

// ---- bits of the device fault word (cvq_fault_status) ----
constexpr unsigned int kFaultCopyTimeout = CVQ_FAULT_COPY_TIMEOUT;   // a TMA copy did not land in time
constexpr unsigned int kFaultBounds = CVQ_FAULT_BOUNDS;             // a debug range check failed

// Range check of the debug build (compiled with -DCVQ_DEBUG_BOUNDS): true if i < n;
// otherwise it sets kFaultBounds in the fault word and returns false, and the caller skips
// the access (a load yields 0) and runs on, so that every barrier is still met.  It never
// traps.  In the regular build it is always true and compiles away.
__device__ __forceinline__ bool in_bounds(unsigned int* fault, size_t i, size_t n) {
#ifdef CVQ_DEBUG_BOUNDS
  if (i < n) return true;
  atomicOr(fault, kFaultBounds);
  return false;
#else
  (void)fault; (void)i; (void)n;
  return true;
#endif
}

constexpr int kCodeBoxRows = 32;   // codes per TMA box of the codebook maps

// ---- mbarrier + TMA (bulk copy engine) helpers ----
// A bounded wait polls the barrier with try_wait, which may suspend the thread until the
// phase completes or for about kMbarSuspendHintNs, and gives up once kMbarWaitLimitNs of
// %globaltimer have passed since its first poll.
constexpr unsigned long long kMbarWaitLimitNs = 2000000000ull;   // 2 s
constexpr unsigned int kMbarSuspendHintNs = 100000u;              // 100 us per poll at most

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// arrive once and add `bytes` to the transaction count the current phase waits for
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned int bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// Wait (bounded) for the completion of the phase with the given parity; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned int parity) {
  const uint32_t addr = smem_u32(bar);
  unsigned long long t0 = 0;
  for (int i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(addr), "r"(parity), "r"(kMbarSuspendHintNs)
        : "memory");
    if (done) return true;
    unsigned long long now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    if (i == 0) t0 = now;
    else if (now - t0 > kMbarWaitLimitNs) return false;
  }
}
// order this thread's earlier generic-proxy shared-memory accesses before later TMA writes
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// 4-d tiled tensor copy, global -> this CTA's shared memory, completing on `bar`
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            int c3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}
// contiguous bulk copy, global -> this CTA's shared memory (both addresses 16-byte aligned,
// bytes a multiple of 16), completing on `bar`
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned int bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The split merge of cvq_combine, fused into the end of a decode kernel.  Every CTA of a
// work unit (sequence b, grid row `unit` = blockIdx.y) calls this with all its threads
// after writing its partial states; `expected` CTAs write the unit's partials.  The CTA
// that arrives last merges the unit's n_heads query heads (hq0 ..) into out and lse with
// the arithmetic of combine_kernel, in the same order, and clears the counter for the
// next call.  No CTA waits for another: the others simply finish.  The arrival is one
// acq_rel atomic per CTA (measured 0.5-1 us faster than a full fence before a relaxed one).
// W warps per query head (n_heads * W <= blockDim / 32): lane l of the head's warp w owns
// the 4 / W output dims 32 w + l + 32 W j and sums them over the splits in split order, as
// combine_kernel does per dim, so both give the same bits; loads go U splits at a time, one
// group ahead of their use.
template <int W = 1, int U = 4>
__device__ __forceinline__ void merge_tail(const DecodeArgs& a, int b, int unit, int hq0,
                                           int n_heads, int expected) {
  static_assert(W == 1 || W == 2 || W == 4, "warps per head");
  constexpr int D = 4 / W;                         // output dims per lane
  const size_t ctr_i = static_cast<size_t>(b) * gridDim.y + unit;
  const bool ctr_ok = in_bounds(a.fault, ctr_i, static_cast<size_t>(a.batch) * a.n_q_heads);
  int* ctr = a.counters + (ctr_ok ? ctr_i : 0);
  int old = 0;
  __syncthreads();                       // this CTA's partial states are all written
  if (threadIdx.x == 0 && ctr_ok) {
    // release: the CTA's partials (ordered before this by the barrier) are visible at GPU
    // scope before the count; acquire: the last CTA then sees every other CTA's partials
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(ctr) : "memory");
  }
  if (!__syncthreads_or(threadIdx.x == 0 && old == expected - 1)) return;
  constexpr int kU = U;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.n_splits;
  const int wl = warp % W;
  for (int hh = warp / W; hh < n_heads; hh += (blockDim.x >> 5) / W) {
    const size_t row = static_cast<size_t>(b) * a.n_q_heads + hq0 + hh;
    if (!in_bounds(a.fault, row, static_cast<size_t>(a.batch) * a.n_q_heads)) continue;
    const float* pm = a.part_m + row * S;
    const float* pl = a.part_l + row * S;
    const float* po = a.part_o + row * S * kHeadDim + 32 * wl + lane;
    float x[kU][D];
    auto load_o = [&](int s0) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
#pragma unroll
        for (int j = 0; j < D; ++j)
          x[u][j] = s0 + u < S ? __ldcg(po + static_cast<size_t>(s0 + u) * kHeadDim + 32 * W * j) : 0.f;
      }
    };
    float mv = lane < S ? __ldcg(pm + lane) : -INFINITY;    // splits 0..31
    float lv = lane < S ? __ldcg(pl + lane) : 0.f;
    load_o(0);
    float M = mv;
    for (int s = lane + 32; s < S; s += 32) M = fmaxf(M, __ldcg(pm + s));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float* orow = a.out + row * kHeadDim + 32 * wl + lane;
    if (M == -INFINITY) {
#pragma unroll
      for (int j = 0; j < D; ++j) orow[32 * W * j] = 0.f;
      if (wl == 0 && lane == 0) a.lse[row] = -INFINITY;
      continue;
    }
    float L = 0.f, acc[D];
#pragma unroll
    for (int j = 0; j < D; ++j) acc[j] = 0.f;
    for (int s0 = 0; s0 < S; s0 += kU) {                      // splits in order
      if (s0 % 32 == 0 && s0 > 0) {                          // next 32 splits' m and l
        mv = s0 + lane < S ? __ldcg(pm + s0 + lane) : -INFINITY;
        lv = s0 + lane < S ? __ldcg(pl + s0 + lane) : 0.f;
      }
      const float fv = (mv == -INFINITY) ? 0.f : expf(mv - M);
      float y[kU][D];
#pragma unroll
      for (int u = 0; u < kU; ++u)
#pragma unroll
        for (int j = 0; j < D; ++j) y[u][j] = x[u][j];
      if (s0 + kU < S) load_o(s0 + kU);                       // the next group, in flight
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (s0 + u < S) {
          const int src = (s0 + u) & 31;
          const float f = __shfl_sync(0xffffffffu, fv, src);
          L = fmaf(__shfl_sync(0xffffffffu, lv, src), f, L);
#pragma unroll
          for (int j = 0; j < D; ++j) acc[j] = fmaf(y[u][j], f, acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < D; ++j) orow[32 * W * j] = acc[j] / L;
    if (wl == 0 && lane == 0) a.lse[row] = M + logf(L);
  }
  if (threadIdx.x == 0 && ctr_ok) atomicExch(ctr, 0);
}

// Launchers (defined next to their kernels).  Return cudaSuccess or the launch error.
cudaError_t launch_qtable(const cvq_shape& s, const void* q, int q_dtype, const float* key_cb,
                          long long key_cb_stride, float* ptable, cudaStream_t stream);
cudaError_t launch_decode_table(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_gqa(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream);
// the clustered kernel for 4 query heads per KV head (decode_gqa.cu)
cudaError_t launch_decode_gqa4(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream);
// the naive baseline (naive.cu, naive_decode.cu)
cudaError_t launch_naive_dequant(const cvq_shape& s, const float* key_cb, long long key_stride,
                                 const float* val_cb, long long val_stride,
                                 const uint8_t* key_codes, const uint8_t* val_codes,
                                 const int32_t* seq_lens, const PhaseTurns& phase, void* k_out,
                                 void* v_out, cudaStream_t stream);
cudaError_t launch_naive_decode(const cvq_shape& s, const void* q, int q_dtype, const void* k,
                                const void* v, const int32_t* seq_lens, int n_splits,
                                int split_tokens, float* part_o, float* part_m, float* part_l,
                                cudaStream_t stream);
// 64-scalar groups, 4 query heads per KV head (decode_wide.cu)
cudaError_t launch_decode_wide(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream);

// The dynamic-shared-memory limit of a kernel is a per-device setting: apply it once per
// (kernel, device) instead of on every launch.  `flag` is a static of the calling launcher,
// one per kernel; devices 0..127.
class PerDeviceFlag {
 public:
  bool done(int dev) const {
    return dev >= 0 && dev < 128 && ((bits_[dev >> 6].load(std::memory_order_acquire) >> (dev & 63)) & 1u);
  }
  void mark(int dev) {
    if (dev >= 0 && dev < 128) bits_[dev >> 6].fetch_or(1ull << (dev & 63), std::memory_order_release);
  }

 private:
  std::atomic<unsigned long long> bits_[2] = {};
};

template <typename Kernel>
cudaError_t set_smem_limit_once(PerDeviceFlag& flag, Kernel kernel, size_t bytes) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (flag.done(dev)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) flag.mark(dev);
  return e;
}

// Host side of the TMA staging and the fault word (device_state.cu).
// Tiled map of one codebook tensor (key or value, narrow layout: per head [16 groups][R][256
// codes][8 floats], heads head_stride floats apart, 0 = one codebook for all heads) whose
// box is 8 groups x kCodeBoxRows codes of one round, landing as [code][local group][8
// floats] (16-byte chunk (code * 8 + local group) * 2 + half).
cudaError_t encode_codebook_map(CUtensorMap* map, const float* base, long long head_stride,
                                int n_heads, int R);
cudaError_t fault_word_address(unsigned int** out);
// the write side: greedy residual encoding of one new key / value per (sequence, KV head)
cudaError_t launch_encode_append(const cvq_shape& s, const float* keys, const float* values,
                                 const float* key_cb, long long key_stride, const float* val_cb,
                                 long long val_stride, const int32_t* positions,
                                 uint8_t* key_codes, uint8_t* val_codes, cudaStream_t stream);
// cvq_attend with its two workspace parts given separately: the split partial states
// (cvq_partials_bytes, 16-byte aligned) and one int32 arrival counter per (sequence, query
// head), which must be zero when the kernel starts.  clear_counters > 0: once every
// argument has passed its checks, first clear that many counters with an asynchronous
// memset on `stream` (api.cu).
cvq_status attend_into(const cvq_shape* s, const void* q, int q_dtype, const float* key_cb,
                       int64_t key_cb_head_stride, const uint8_t* key_codes,
                       const uint8_t* val_codes, const int32_t* seq_lens, const float* val_cb,
                       int64_t val_cb_head_stride, int n_splits, float* partials, int* counters,
                       float* out, float* lse, void* stream, size_t clear_counters);
// 6-bit packing of `rows` planar code rows of t_cap codes each (pack.cu)
cudaError_t launch_pack_codes6(const uint8_t* codes_in, uint8_t* packed_out, size_t rows, int t_cap,
                               cudaStream_t stream);
cudaError_t launch_combine(const cvq_shape& s, int n_splits, const float* part_o,
                           const float* part_m, const float* part_l, float* out, float* lse,
                           cudaStream_t stream);

}  // namespace cvq
