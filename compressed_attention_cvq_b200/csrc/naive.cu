// The naive path that CommVQ is compared against (CommVQ summary page, "Key results" and
// "Measured effects": the optimized commutative-codebook implementation versus the naive
// implementation): first decode every cached key and value from its codes into fp16 in
// HBM -- keys reconstructed and rotated by RoPE -- then run ordinary split-T decode
// attention over the fp16 cache.
//
// naive_dequant_kernel: one thread per (token, group); the thread sums the R key codewords
// of its 4 pairs, rotates them by the exact phase of position t and stores 8 fp16 key dims,
// then sums the R value codewords and stores 8 fp16 value dims.
// The attention half is naive_decode.cu; naive_dequant_wide_kernel below does the paper's
// layout.
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
  // F_j from shared memory: the 16 groups of a warp read 16 different pairs, and an indexed
  // read of the parameter space serializes over distinct addresses
  __shared__ unsigned long long f_tab[kPairs];
  for (int i = threadIdx.x; i < kPairs; i += kDqThreads) f_tab[i] = phase.F[i];
  __syncthreads();
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
    const float2 ph = phase_at(f_tab[4 * G + p], t);
    ko[p] = __floats2half2_rn(ph.x * kr[p] - ph.y * ki[p], ph.y * kr[p] + ph.x * ki[p]);
    vo[p] = __floats2half2_rn(v[2 * p], v[2 * p + 1]);
  }
  *reinterpret_cast<uint4*>(k_out + row * kHeadDim + 8 * G) = *reinterpret_cast<uint4*>(ko);
  *reinterpret_cast<uint4*>(v_out + row * kHeadDim + 8 * G) = *reinterpret_cast<uint4*>(vo);
}

// The same for the paper's layout (2 groups of 64 scalars, 64 codewords, planar codes
// [B, Hkv, 2, R, t_cap], or packed 6-bit rows of 3 t_cap / 4 bytes when packed6): block
// (32 tokens, 8 chunks) per (token block, KV head x group,
// sequence); thread (token, chunk) sums the R codewords' 8-float chunk of its group for
// the key (pairs 32 G + 4 chunk .. + 3, rotated) and the value (dims 64 G + 8 chunk ..).
__global__ void __launch_bounds__(256) naive_dequant_wide_kernel(
    const float* __restrict__ key_cb, long long key_stride, const float* __restrict__ val_cb,
    long long val_stride, const uint8_t* __restrict__ key_codes,
    const uint8_t* __restrict__ val_codes, const int32_t* __restrict__ seq_lens, int R,
    int n_kv_heads, int t_cap, PhaseTurns phase, __half* __restrict__ k_out,
    __half* __restrict__ v_out, bool packed6) {
  __shared__ unsigned long long f_tab[kPairs];      // F_j, as in naive_dequant_kernel
  for (int i = threadIdx.y * 32 + threadIdx.x; i < kPairs; i += 256) f_tab[i] = phase.F[i];
  __syncthreads();
  const int t = blockIdx.x * 32 + threadIdx.x;
  const int chunk = threadIdx.y;
  const int G = blockIdx.y & 1, h = blockIdx.y >> 1, b = blockIdx.z;
  int L = seq_lens[b];
  L = L < 0 ? 0 : (L > t_cap ? t_cap : L);
  if (t >= L) return;
  const size_t bh = static_cast<size_t>(b) * n_kv_heads + h;
  const size_t row_bytes = packed6 ? static_cast<size_t>(t_cap) / 4 * 3 : static_cast<size_t>(t_cap);
  const uint8_t* kc = key_codes + (bh * kWideGroups + G) * R * row_bytes;
  const uint8_t* vc = val_codes + (bh * kWideGroups + G) * R * row_bytes;
  const float* kcb = key_cb + h * key_stride + static_cast<size_t>(G) * R * kWideCodes * kWideVDims + 8 * chunk;
  const float* vcb = val_cb + h * val_stride + static_cast<size_t>(G) * R * kWideCodes * kWideVDims + 8 * chunk;
  float k[8], v[8];
#pragma unroll
  for (int d = 0; d < 8; ++d) k[d] = v[d] = 0.f;
  for (int r = 0; r < R; ++r) {
    const uint8_t* krow = kc + static_cast<size_t>(r) * row_bytes;
    const uint8_t* vrow = vc + static_cast<size_t>(r) * row_bytes;
    const int ck = packed6 ? packed6_code(krow, t) : (krow[t] & (kWideCodes - 1));
    const int cv = packed6 ? packed6_code(vrow, t) : (vrow[t] & (kWideCodes - 1));
    const float4* kw = reinterpret_cast<const float4*>(kcb + (static_cast<size_t>(r) * kWideCodes + ck) * kWideVDims);
    const float4* vw = reinterpret_cast<const float4*>(vcb + (static_cast<size_t>(r) * kWideCodes + cv) * kWideVDims);
    const float4 a0 = __ldg(kw), a1 = __ldg(kw + 1), b0 = __ldg(vw), b1 = __ldg(vw + 1);
    k[0] += a0.x; k[1] += a0.y; k[2] += a0.z; k[3] += a0.w;
    k[4] += a1.x; k[5] += a1.y; k[6] += a1.z; k[7] += a1.w;
    v[0] += b0.x; v[1] += b0.y; v[2] += b0.z; v[3] += b0.w;
    v[4] += b1.x; v[5] += b1.y; v[6] += b1.z; v[7] += b1.w;
  }
  __half2 ko[4], vo[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 ph = phase_at(f_tab[kWidePairs * G + 4 * chunk + p], t);
    ko[p] = __floats2half2_rn(ph.x * k[2 * p] - ph.y * k[2 * p + 1],
                              ph.y * k[2 * p] + ph.x * k[2 * p + 1]);
    vo[p] = __floats2half2_rn(v[2 * p], v[2 * p + 1]);
  }
  const size_t o = (bh * t_cap + t) * kHeadDim + kWideVDims * G + 8 * chunk;
  *reinterpret_cast<uint4*>(k_out + o) = *reinterpret_cast<uint4*>(ko);
  *reinterpret_cast<uint4*>(v_out + o) = *reinterpret_cast<uint4*>(vo);
}

}  // namespace

cudaError_t launch_naive_dequant(const cvq_shape& s, const float* key_cb, long long key_stride,
                                 const float* val_cb, long long val_stride,
                                 const uint8_t* key_codes, const uint8_t* val_codes,
                                 const int32_t* seq_lens, const PhaseTurns& phase, void* k_out,
                                 void* v_out, cudaStream_t stream) {
  if (s.t_cap == 0) return cudaSuccess;
  if (s.group_dim == kWideGroupDim) {
    dim3 grid((s.t_cap + 31) / 32, s.n_kv_heads * kWideGroups, s.batch);
    naive_dequant_wide_kernel<<<grid, dim3(32, 8), 0, stream>>>(
        key_cb, key_stride, val_cb, val_stride, key_codes, val_codes, seq_lens, s.R,
        s.n_kv_heads, s.t_cap, phase, static_cast<__half*>(k_out), static_cast<__half*>(v_out),
        s.code_bits == 6);
    return cudaGetLastError();
  }
  dim3 grid((s.t_cap + kDqThreads / 16 - 1) / (kDqThreads / 16), s.n_kv_heads, s.batch);
  naive_dequant_kernel<<<grid, kDqThreads, 0, stream>>>(
      key_cb, key_stride, val_cb, val_stride, key_codes, val_codes, seq_lens, s.R, s.n_kv_heads,
      s.t_cap, phase, static_cast<__half*>(k_out), static_cast<__half*>(v_out));
  return cudaGetLastError();
}

}  // namespace cvq
