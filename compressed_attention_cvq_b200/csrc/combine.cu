// cvq_combine: log-sum-exp merge of split-T partial states into out and lse.
//   M = max_s m_s;  L = sum_s l_s e^{m_s - M};  out = sum_s o_s e^{m_s - M} / L;
//   lse = M + ln L;  every split empty -> out = 0, lse = -inf.
// One CTA of 128 threads per (b, hq); thread d owns output dim d.  The split scale
// factors are computed once per CTA into shared memory.
#include "common.cuh"

namespace cvq {

constexpr int kCombineThreads = 128;
constexpr int kCombineChunk = 512;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_m,
    const float* __restrict__ part_l, float* __restrict__ out, float* __restrict__ lse,
    int n_splits) {
  __shared__ float scale[kCombineChunk];
  __shared__ float red[kCombineThreads / 32];
  const int row = blockIdx.x;                 // b * Hq + hq
  const int tid = threadIdx.x;
  const float* pm = part_m + static_cast<size_t>(row) * n_splits;
  const float* pl = part_l + static_cast<size_t>(row) * n_splits;
  const float* po = part_o + static_cast<size_t>(row) * n_splits * kHeadDim;

  float M = -INFINITY;
  for (int s = tid; s < n_splits; s += kCombineThreads) M = fmaxf(M, pm[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (tid % 32 == 0) red[tid / 32] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < kCombineThreads / 32; ++w) M = fmaxf(M, red[w]);
  __syncthreads();

  if (M == -INFINITY) {
    out[static_cast<size_t>(row) * kHeadDim + tid] = 0.f;
    if (tid == 0) lse[row] = -INFINITY;
    return;
  }
  float L = 0.f, acc = 0.f;
  for (int s0 = 0; s0 < n_splits; s0 += kCombineChunk) {
    const int n = min(kCombineChunk, n_splits - s0);
    for (int i = tid; i < n; i += kCombineThreads) {
      const float m = pm[s0 + i];
      scale[i] = (m == -INFINITY) ? 0.f : expf(m - M);
    }
    __syncthreads();
    for (int i = 0; i < n; ++i) {
      const float f = scale[i];
      L = fmaf(pl[s0 + i], f, L);
      acc = fmaf(po[static_cast<size_t>(s0 + i) * kHeadDim + tid], f, acc);
    }
    __syncthreads();
  }
  out[static_cast<size_t>(row) * kHeadDim + tid] = acc / L;
  if (tid == 0) lse[row] = M + logf(L);
}

cudaError_t launch_combine(const cvq_shape& s, int n_splits, const float* part_o,
                           const float* part_m, const float* part_l, float* out, float* lse,
                           cudaStream_t stream) {
  combine_kernel<<<static_cast<unsigned>(s.batch) * s.n_q_heads, kCombineThreads, 0, stream>>>(
      part_o, part_m, part_l, out, lse, n_splits);
  return cudaGetLastError();
}

}  // namespace cvq
