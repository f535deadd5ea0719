// cvq_encode_append: write the codes of one new key and value per (sequence, KV head) at
// position positions[b] of the code cache -- the write side of a decode step.
//
// The pages encode with a learned encoder (CommVQ abstract; summary page "Approach"),
// which needs trained weights; this is greedy additive quantization instead: for each
// group and residual round (review page, "key_machinery": R rounds refine the
// reconstruction) take the codeword nearest to the current residual and subtract it.
// Keys are encoded before RoPE, as the cache stores them.
//
// One CTA per (sequence x KV head, group, key | value); thread c scores codeword c.  The
// squared distance is summed in float32 in dim order 0..7 with no fused multiply-add, and
// ties go to the smaller code, so the chosen code is a fixed function of the inputs.
#include "common.cuh"

namespace cvq {

namespace {

__global__ void __launch_bounds__(kCodes) encode_kernel(
    const float* __restrict__ keys, const float* __restrict__ values,
    const float* __restrict__ key_cb, long long key_stride, const float* __restrict__ val_cb,
    long long val_stride, const int32_t* __restrict__ positions, uint8_t* __restrict__ key_codes,
    uint8_t* __restrict__ val_codes, int R, int n_kv_heads, int t_cap) {
  __shared__ float res[8];
  __shared__ float best_d[kCodes / 32];
  __shared__ int best_c[kCodes / 32];
  __shared__ int chosen;
  const int bh = blockIdx.x, G = blockIdx.y, is_val = blockIdx.z;
  const int b = bh / n_kv_heads, h = bh % n_kv_heads;
  const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
  const int p = positions[b];
  if (p < 0 || p >= t_cap) return;                       // uniform for the CTA
  const float* src = (is_val ? values : keys) + static_cast<size_t>(bh) * kHeadDim + 8 * G;
  const float* cb = is_val ? val_cb + h * val_stride : key_cb + h * key_stride;
  uint8_t* out = (is_val ? val_codes : key_codes) +
                 ((static_cast<size_t>(bh) * t_cap + p) * R) * 16 + G;
  if (c < 8) res[c] = src[c];
  __syncthreads();
  for (int r = 0; r < R; ++r) {
    const float4* cw = reinterpret_cast<const float4*>(cb + ((static_cast<size_t>(G) * R + r) * kCodes + c) * 8);
    const float4 lo = __ldg(cw), hi = __ldg(cw + 1);
    const float w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    float acc = 0.f;
#pragma unroll
    for (int d = 0; d < 8; ++d) {
      const float diff = __fsub_rn(res[d], w[d]);
      acc = __fadd_rn(acc, __fmul_rn(diff, diff));
    }
    // arg-min over the 256 codewords, smaller code on ties
    float bd = acc;
    int bc = c;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, bd, o);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      if (od < bd || (od == bd && oc < bc)) { bd = od; bc = oc; }
    }
    if (lane == 0) { best_d[warp] = bd; best_c[warp] = bc; }
    __syncthreads();
    if (c == 0) {
      float d0 = best_d[0];
      int c0 = best_c[0];
      for (int i = 1; i < kCodes / 32; ++i) {
        if (best_d[i] < d0 || (best_d[i] == d0 && best_c[i] < c0)) { d0 = best_d[i]; c0 = best_c[i]; }
      }
      chosen = c0;
      out[r * 16] = static_cast<uint8_t>(c0);
    }
    __syncthreads();
    if (c < 8) res[c] = __fsub_rn(res[c], cb[((static_cast<size_t>(G) * R + r) * kCodes + chosen) * 8 + c]);
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_encode_append(const cvq_shape& s, const float* keys, const float* values,
                                 const float* key_cb, long long key_stride, const float* val_cb,
                                 long long val_stride, const int32_t* positions,
                                 uint8_t* key_codes, uint8_t* val_codes, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(s.batch) * s.n_kv_heads, kGroups, 2);
  encode_kernel<<<grid, kCodes, 0, stream>>>(keys, values, key_cb, key_stride, val_cb, val_stride,
                                             positions, key_codes, val_codes, s.R, s.n_kv_heads,
                                             s.t_cap);
  return cudaGetLastError();
}

}  // namespace cvq
