// Decode attention over the fp16 keys / values written by naive_dequant_kernel (the naive
// path's second half).  One CTA per (split, KV head, sequence) for its NG query heads.
// 16 lanes per token, each lane 8 dims (one 16-byte load of K and of V); the partial dot
// products are summed over the 16 lanes with shuffles; every 16-lane group keeps its own
// online-softmax state for its token stream, merged across streams in shared memory at
// the end.  m is the exact split maximum.  With 8 dims per lane the 4-head kernel holds
// its queries and accumulators in ~100 registers, so two CTAs fit an SM.
#include <cuda_fp16.h>

#include "common.cuh"

namespace cvq {

namespace {

constexpr int kNvThreads = 256;                 // 8 warps x 2 token streams
constexpr int kLanesPerToken = 16;
constexpr int kDimsPerLane = kHeadDim / kLanesPerToken;   // 8
constexpr int kStreams = kNvThreads / kLanesPerToken;     // 16 token streams per CTA

template <int NG>
__global__ void __launch_bounds__(kNvThreads, 2) naive_decode_kernel(
    const void* __restrict__ q, int q_dtype, const __half* __restrict__ kc,
    const __half* __restrict__ vc, const int32_t* __restrict__ seq_lens, int n_q_heads,
    int n_kv_heads, int t_cap, int n_splits, int split_tokens, float* __restrict__ part_o,
    float* __restrict__ part_m, float* __restrict__ part_l) {
  extern __shared__ float sm[];                 // [kStreams][NG][128 + 2]
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31;
  const int stream = tid / kLanesPerToken;      // token stream (16 lanes each)
  const int k = lane % kLanesPerToken;          // dims 8k .. 8k + 7
  const int hq0 = h * NG;
  int L = seq_lens[b];
  L = L < 0 ? 0 : (L > t_cap ? t_cap : L);
  const int t_begin = split * split_tokens;
  const int t_end = min(t_begin + split_tokens, L);
  const size_t part_row = (static_cast<size_t>(b) * n_q_heads + hq0) * n_splits + split;

  const float qscale = kLog2e * 0.08838834764831845f;
  float qv[NG][kDimsPerLane];
#pragma unroll
  for (int hh = 0; hh < NG; ++hh) {
#pragma unroll
    for (int d = 0; d < kDimsPerLane; ++d)
      qv[hh][d] = load_q(q, q_dtype, (static_cast<size_t>(b) * n_q_heads + hq0 + hh) * kHeadDim +
                                         kDimsPerLane * k + d) * qscale;
  }
  float m[NG], l[NG], o[NG][kDimsPerLane];
#pragma unroll
  for (int hh = 0; hh < NG; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int d = 0; d < kDimsPerLane; ++d) o[hh][d] = 0.f;
  }
  const size_t row0 = (static_cast<size_t>(b) * n_kv_heads + h) * t_cap;
  // the 16 lanes of a stream run the same number of iterations, but the streams of one warp
  // may not (tail of the split): shuffles name only the stream's own lanes
  const unsigned gmask = 0xffffu << (lane & 16);
  for (int t = t_begin + stream; t < t_end; t += kStreams) {
    const uint4 k0 = __ldg(reinterpret_cast<const uint4*>(kc + (row0 + t) * kHeadDim + kDimsPerLane * k));
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(vc + (row0 + t) * kHeadDim + kDimsPerLane * k));
    const __half2* kh0 = reinterpret_cast<const __half2*>(&k0);
    const __half2* vh0 = reinterpret_cast<const __half2*>(&v0);
    float kf[kDimsPerLane], vf[kDimsPerLane];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 a = __half22float2(kh0[i]);
      kf[2 * i] = a.x; kf[2 * i + 1] = a.y;
      a = __half22float2(vh0[i]);
      vf[2 * i] = a.x; vf[2 * i + 1] = a.y;
    }
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) {
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < kDimsPerLane; ++d) s = fmaf(qv[hh][d], kf[d], s);
      s += __shfl_xor_sync(gmask, s, 1);
      s += __shfl_xor_sync(gmask, s, 2);
      s += __shfl_xor_sync(gmask, s, 4);
      s += __shfl_xor_sync(gmask, s, 8);
      const float m_new = fmaxf(m[hh], s);
      const float f = exp2f(m[hh] - m_new);   // 0 on the first token (m = -inf)
      const float w = exp2f(s - m_new);
      l[hh] = l[hh] * f + w;
#pragma unroll
      for (int d = 0; d < kDimsPerLane; ++d) o[hh][d] = fmaf(o[hh][d], f, w * vf[d]);
      m[hh] = m_new;
    }
  }
  // merge the 32 token streams: stream state -> shared memory -> per (head, dim) merge
  float* st = sm + static_cast<size_t>(stream) * NG * (kHeadDim + 2);
#pragma unroll
  for (int hh = 0; hh < NG; ++hh) {
#pragma unroll
    for (int d = 0; d < kDimsPerLane; ++d) st[hh * (kHeadDim + 2) + kDimsPerLane * k + d] = o[hh][d];
    if (k == 0) {
      st[hh * (kHeadDim + 2) + kHeadDim] = m[hh];
      st[hh * (kHeadDim + 2) + kHeadDim + 1] = l[hh];
    }
  }
  __syncthreads();
  for (int i = tid; i < NG * kHeadDim; i += kNvThreads) {
    const int hh = i / kHeadDim, d = i % kHeadDim;
    float M = -INFINITY;
    for (int s2 = 0; s2 < kStreams; ++s2) M = fmaxf(M, sm[(s2 * NG + hh) * (kHeadDim + 2) + kHeadDim]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < kStreams; ++s2) {
        const float* e = sm + (s2 * NG + hh) * (kHeadDim + 2);
        const float f = exp2f(e[kHeadDim] - M);
        acc = fmaf(e[d], f, acc);
        lsum = fmaf(e[kHeadDim + 1], f, lsum);
      }
    }
    part_o[(part_row + static_cast<size_t>(hh) * n_splits) * kHeadDim + d] = acc;
    if (d == 0) {
      part_m[part_row + static_cast<size_t>(hh) * n_splits] = (M == -INFINITY) ? -INFINITY : M * kLn2;
      part_l[part_row + static_cast<size_t>(hh) * n_splits] = lsum;
    }
  }
}

template <int NG>
cudaError_t launch_nv(const cvq_shape& s, const void* q, int q_dtype, const void* k, const void* v,
                      const int32_t* seq_lens, int n_splits, int split_tokens, float* po,
                      float* pm, float* pl, cudaStream_t stream) {
  const size_t smem = sizeof(float) * kStreams * NG * (kHeadDim + 2);
  auto kern = naive_decode_kernel<NG>;
  static PerDeviceFlag smem_set;
  cudaError_t e = set_smem_limit_once(smem_set, kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_splits, s.n_kv_heads, s.batch);
  kern<<<grid, kNvThreads, smem, stream>>>(q, q_dtype, static_cast<const __half*>(k),
                                           static_cast<const __half*>(v), seq_lens, s.n_q_heads,
                                           s.n_kv_heads, s.t_cap, n_splits, split_tokens, po, pm,
                                           pl);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_naive_decode(const cvq_shape& s, const void* q, int q_dtype, const void* k,
                                const void* v, const int32_t* seq_lens, int n_splits,
                                int split_tokens, float* part_o, float* part_m, float* part_l,
                                cudaStream_t stream) {
  switch (s.n_q_heads / s.n_kv_heads) {
    case 1: return launch_nv<1>(s, q, q_dtype, k, v, seq_lens, n_splits, split_tokens, part_o, part_m, part_l, stream);
    case 2: return launch_nv<2>(s, q, q_dtype, k, v, seq_lens, n_splits, split_tokens, part_o, part_m, part_l, stream);
    case 4: return launch_nv<4>(s, q, q_dtype, k, v, seq_lens, n_splits, split_tokens, part_o, part_m, part_l, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace cvq
