// The naive path that CommVQ is compared against (CommVQ summary page, "Key results" and
// "Measured effects": the optimized commutative-codebook implementation versus the naive
// implementation): first decode every cached key and value from its codes into fp16 in
// HBM -- keys reconstructed and rotated by RoPE -- then run ordinary split-T decode
// attention over the fp16 cache.
//
// naive_dequant_kernel: one thread per (token, group); the thread sums the R key codewords
// of its 4 pairs, rotates them by the exact phase of position t and stores 8 fp16 key dims,
// then sums the R value codewords and stores 8 fp16 value dims.
// The attention half is naive_decode.cu.
#include <cuda_fp16.h>

#include "common.cuh"

namespace cvq {

namespace {

constexpr int kDqThreads = 256;   // 16 tokens x 16 groups

__global__ void __launch_bounds__(kDqThreads) naive_dequant_kernel(
    const float* __restrict__ key_cb, long long key_stride, const float* __restrict__ val_cb,
    long long val_stride, const uint8_t* __restrict__ key_codes,
    const uint8_t* __restrict__ val_codes, const int32_t* __restrict__ seq_lens, int R,
    int n_kv_heads, int t_cap, PhaseTurns phase, __half* __restrict__ k_out,
    __half* __restrict__ v_out) {
  const int G = threadIdx.x & 15;
  const int t = blockIdx.x * (kDqThreads / 16) + (threadIdx.x >> 4);
  const int h = blockIdx.y, b = blockIdx.z;
  int L = seq_lens[b];
  L = L < 0 ? 0 : (L > t_cap ? t_cap : L);
  if (t >= L) return;
  const size_t row = (static_cast<size_t>(b) * n_kv_heads + h) * t_cap + t;
  const uint8_t* kc = key_codes + row * (16 * R);
  const uint8_t* vc = val_codes + row * (16 * R);
  const float* kcb = key_cb + h * key_stride;
  const float* vcb = val_cb + h * val_stride;
  float kr[4] = {0.f, 0.f, 0.f, 0.f}, ki[4] = {0.f, 0.f, 0.f, 0.f}, v[8];
#pragma unroll
  for (int d = 0; d < 8; ++d) v[d] = 0.f;
  for (int r = 0; r < R; ++r) {
    const int ck = kc[r * 16 + G], cv = vc[r * 16 + G];
    const float4* kw = reinterpret_cast<const float4*>(kcb + ((static_cast<size_t>(G) * R + r) * kCodes + ck) * kCodeword);
    const float4 a0 = __ldg(kw), a1 = __ldg(kw + 1);
    kr[0] += a0.x; ki[0] += a0.y; kr[1] += a0.z; ki[1] += a0.w;
    kr[2] += a1.x; ki[2] += a1.y; kr[3] += a1.z; ki[3] += a1.w;
    const float4* vw = reinterpret_cast<const float4*>(vcb + ((static_cast<size_t>(G) * R + r) * kCodes + cv) * kVDims);
    const float4 b0 = __ldg(vw), b1 = __ldg(vw + 1);
    v[0] += b0.x; v[1] += b0.y; v[2] += b0.z; v[3] += b0.w;
    v[4] += b1.x; v[5] += b1.y; v[6] += b1.z; v[7] += b1.w;
  }
  __half2 ko[4], vo[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 ph = phase_at(phase.F[4 * G + p], t);
    ko[p] = __floats2half2_rn(ph.x * kr[p] - ph.y * ki[p], ph.y * kr[p] + ph.x * ki[p]);
    vo[p] = __floats2half2_rn(v[2 * p], v[2 * p + 1]);
  }
  *reinterpret_cast<uint4*>(k_out + row * kHeadDim + 8 * G) = *reinterpret_cast<uint4*>(ko);
  *reinterpret_cast<uint4*>(v_out + row * kHeadDim + 8 * G) = *reinterpret_cast<uint4*>(vo);
}

}  // namespace

cudaError_t launch_naive_dequant(const cvq_shape& s, const float* key_cb, long long key_stride,
                                 const float* val_cb, long long val_stride,
                                 const uint8_t* key_codes, const uint8_t* val_codes,
                                 const int32_t* seq_lens, const PhaseTurns& phase, void* k_out,
                                 void* v_out, cudaStream_t stream) {
  if (s.t_cap == 0) return cudaSuccess;
  dim3 grid((s.t_cap + kDqThreads / 16 - 1) / (kDqThreads / 16), s.n_kv_heads, s.batch);
  naive_dequant_kernel<<<grid, kDqThreads, 0, stream>>>(
      key_cb, key_stride, val_cb, val_stride, key_codes, val_codes, seq_lens, s.R, s.n_kv_heads,
      s.t_cap, phase, static_cast<__half*>(k_out), static_cast<__half*>(v_out));
  return cudaGetLastError();
}

}  // namespace cvq
