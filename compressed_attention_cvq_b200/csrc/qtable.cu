// cvq_qtable: P[b, hq, G, r, c, p] = conj(q_j) * c  (j = 4G + p), the query x
// key-codebook table of the CommVQ review page ("key_machinery": the query-dependent
// and codebook-dependent factors are combined once per query).
//
// One CTA per (b, hq) x (G, r); one thread per codeword c.  Each thread reads its
// codeword (two 16-byte loads), multiplies by the 4 conjugated query pairs of group G
// and writes 32 contiguous bytes, so a warp stores 1 KB contiguously.
#include "common.cuh"

namespace cvq {

__global__ void __launch_bounds__(kCodes) qtable_kernel(const void* __restrict__ q, int q_dtype,
                                                        const float* __restrict__ key_cb,
                                                        long long key_cb_stride,
                                                        float* __restrict__ ptable, int n_q_heads,
                                                        int n_kv_heads, int R) {
  const int bh = blockIdx.x;              // b * Hq + hq
  const int G = blockIdx.y / R;
  const int r = blockIdx.y % R;
  const int c = threadIdx.x;
  const int hq = bh % n_q_heads;
  const int h = hq / (n_q_heads / n_kv_heads);

  float qr[kPairsPerGroup], qi[kPairsPerGroup];
  const size_t qbase = static_cast<size_t>(bh) * kHeadDim + 8 * G;
#pragma unroll
  for (int p = 0; p < kPairsPerGroup; ++p) {
    qr[p] = load_q(q, q_dtype, qbase + 2 * p);
    qi[p] = load_q(q, q_dtype, qbase + 2 * p + 1);
  }
  const size_t cw = (static_cast<size_t>(G) * R + r) * kCodes + c;
  const float4* src = reinterpret_cast<const float4*>(key_cb + h * key_cb_stride + cw * kCodeword);
  const float4 lo = __ldg(src), hi = __ldg(src + 1);
  const float a[4] = {lo.x, lo.z, hi.x, hi.z};
  const float bb[4] = {lo.y, lo.w, hi.y, hi.w};
  float o[8];
#pragma unroll
  for (int p = 0; p < kPairsPerGroup; ++p) {
    // (qr - i qi)(a + i b) = (qr a + qi b) + i (qr b - qi a)
    o[2 * p] = fmaf(qr[p], a[p], qi[p] * bb[p]);
    o[2 * p + 1] = fmaf(qr[p], bb[p], -qi[p] * a[p]);
  }
  float4* dst = reinterpret_cast<float4*>(
      ptable + ((static_cast<size_t>(bh) * kGroups + G) * R + r) * kCodes * kCodeword +
      static_cast<size_t>(c) * kCodeword);
  dst[0] = make_float4(o[0], o[1], o[2], o[3]);
  dst[1] = make_float4(o[4], o[5], o[6], o[7]);
}

cudaError_t launch_qtable(const cvq_shape& s, const void* q, int q_dtype, const float* key_cb,
                          long long key_cb_stride, float* ptable, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(s.batch) * s.n_q_heads, kGroups * s.R);
  qtable_kernel<<<grid, kCodes, 0, stream>>>(q, q_dtype, key_cb, key_cb_stride, ptable,
                                             s.n_q_heads, s.n_kv_heads, s.R);
  return cudaGetLastError();
}

}  // namespace cvq
