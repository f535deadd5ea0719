// cvq_encode_append: write the codes of one new key and value per (sequence, KV head) at
// position positions[b] of the code cache -- the write side of a decode step, for both
// cache layouts (16 groups of 8 scalars; 2 groups of 64 scalars).
//
// The pages encode with a learned encoder (CommVQ abstract; summary page "Approach"),
// which needs trained weights; this is greedy additive quantization instead: for each
// group and residual round (review page, "key_machinery": R rounds refine the
// reconstruction) take the codeword nearest to the current residual and subtract it.
// Keys are encoded before RoPE, as the cache stores them.
//
// One warp per (sequence x KV head, group, key | value); lane l scores codewords
// l, l + 32, ..., l + 224.  The squared distance is summed in float32 in dim order 0..7
// with no fused multiply-add, and ties go to the smaller code, so the chosen code is a
// fixed function of the inputs.  No shared memory and no block barrier: the residual
// lives in every lane's registers, and the winner's codeword reaches the warp by shuffles.
// Every load of the first round (position, input, codewords) is independent of the others
// and issued up front; the next round's codewords are loaded while this round's arg-min
// runs.
#include "common.cuh"

namespace cvq {

namespace {

constexpr int kEncWarps = 8;                   // (group, key | value) units per CTA
constexpr int kPerLane = kCodes / 32;          // codewords scored by each lane

__device__ __forceinline__ void load_round(const float* cb_round, int lane, float4 (&w)[2 * kPerLane]) {
  const float4* p = reinterpret_cast<const float4*>(cb_round) + 2 * lane;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    w[2 * i] = __ldg(p + 64 * i);
    w[2 * i + 1] = __ldg(p + 64 * i + 1);
  }
}

__global__ void __launch_bounds__(32 * kEncWarps) encode_kernel(
    const float* __restrict__ keys, const float* __restrict__ values,
    const float* __restrict__ key_cb, long long key_stride, const float* __restrict__ val_cb,
    long long val_stride, const int32_t* __restrict__ positions, uint8_t* __restrict__ key_codes,
    uint8_t* __restrict__ val_codes, int R, int n_kv_heads, int t_cap) {
  const int lane = threadIdx.x & 31;
  const int unit = blockIdx.x * kEncWarps + (threadIdx.x >> 5);   // (bh, is_val, G)
  const int G = unit & 15, is_val = (unit >> 4) & 1, bh = unit >> 5;
  const int b = bh / n_kv_heads, h = bh % n_kv_heads;
  const float* src = (is_val ? values : keys) + static_cast<size_t>(bh) * kHeadDim + 8 * G;
  const float* cb = (is_val ? val_cb + h * val_stride : key_cb + h * key_stride) +
                    static_cast<size_t>(G) * R * kCodes * 8;

  float4 w[2 * kPerLane];
  load_round(cb, lane, w);
  const float4 x0 = __ldg(reinterpret_cast<const float4*>(src));
  const float4 x1 = __ldg(reinterpret_cast<const float4*>(src) + 1);
  const int p = positions[b];
  if (p < 0 || p >= t_cap) return;                       // uniform for the warp
  uint8_t* out = (is_val ? val_codes : key_codes) +
                 ((static_cast<size_t>(bh) * t_cap + p) * R) * 16 + G;
  float res[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};

  for (int r = 0; r < R; ++r) {
    // this lane's nearest codeword (scanned in ascending code order, strict <)
    float bd = INFINITY;
    int bi = 0;
    float bw[8];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const float c[8] = {w[2 * i].x, w[2 * i].y, w[2 * i].z, w[2 * i].w,
                          w[2 * i + 1].x, w[2 * i + 1].y, w[2 * i + 1].z, w[2 * i + 1].w};
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        const float diff = __fsub_rn(res[d], c[d]);
        acc = __fadd_rn(acc, __fmul_rn(diff, diff));
      }
      const bool better = (i == 0) || (acc < bd);
      bd = better ? acc : bd;
      bi = better ? i : bi;
#pragma unroll
      for (int d = 0; d < 8; ++d) bw[d] = better ? c[d] : bw[d];
    }
    if (r + 1 < R) load_round(cb + static_cast<size_t>(r + 1) * kCodes * 8, lane, w);
    // warp arg-min over (distance, code); code = lane + 32 * i
    float md = bd;
    int mc = lane + 32 * bi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, md, o);
      const int oc = __shfl_xor_sync(0xffffffffu, mc, o);
      if (od < md || (od == md && oc < mc)) { md = od; mc = oc; }
    }
    if (lane == 0) out[r * 16] = static_cast<uint8_t>(mc);
    // residual -= the chosen codeword, held by lane mc & 31
#pragma unroll
    for (int d = 0; d < 8; ++d) res[d] = __fsub_rn(res[d], __shfl_sync(0xffffffffu, bw[d], mc & 31));
  }
}

// The paper's layout: 2 groups of 64 scalars, 64 codewords per (group, round), planar codes
// [B, Hkv, 2, R, t_cap], one byte per code, or (packed6) 4 codes in 3 bytes per row, where
// only the 6 bits of the written code change (a read-modify-write of its one or two bytes;
// no other thread writes the row in the same call).  One warp per (sequence x KV head,
// key | value, group); lane l scores codewords l and l + 32.  The residual (64 floats) sits
// in shared memory and every lane reads it in dim order 0..63, so each distance is summed
// in one fixed order.
constexpr int kWideEncWarps = 8;

__global__ void __launch_bounds__(32 * kWideEncWarps) encode_wide_kernel(
    const float* __restrict__ keys, const float* __restrict__ values,
    const float* __restrict__ key_cb, long long key_stride, const float* __restrict__ val_cb,
    long long val_stride, const int32_t* __restrict__ positions, uint8_t* __restrict__ key_codes,
    uint8_t* __restrict__ val_codes, int R, int n_kv_heads, int t_cap, int n_units, bool packed6) {
  __shared__ __align__(16) float res_s[kWideEncWarps][kWideVDims];
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const int unit = blockIdx.x * kWideEncWarps + wl;             // (bh, is_val, G)
  if (unit >= n_units) return;                                   // uniform for the warp
  const int G = unit & 1, is_val = (unit >> 1) & 1, bh = unit >> 2;
  const int b = bh / n_kv_heads, h = bh % n_kv_heads;
  const int p = positions[b];
  if (p < 0 || p >= t_cap) return;                               // uniform for the warp
  const float* src = (is_val ? values : keys) + static_cast<size_t>(bh) * kHeadDim + kWideVDims * G;
  const float* cb = (is_val ? val_cb + h * val_stride : key_cb + h * key_stride) +
                    static_cast<size_t>(G) * R * kWideCodes * kWideVDims;
  const size_t row_bytes = packed6 ? static_cast<size_t>(t_cap) / 4 * 3 : static_cast<size_t>(t_cap);
  uint8_t* rows = (is_val ? val_codes : key_codes) + ((static_cast<size_t>(bh) * kWideGroups + G) * R) * row_bytes;
  float* res = res_s[wl];
  res[lane] = src[lane];
  res[lane + 32] = src[lane + 32];
  __syncwarp();
  for (int r = 0; r < R; ++r) {
    const float4* c0 = reinterpret_cast<const float4*>(cb + (static_cast<size_t>(r) * kWideCodes + lane) * kWideVDims);
    const float4* c1 = c0 + 32 * kWideVDims / 4;                 // codeword lane + 32
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
    for (int q = 0; q < kWideVDims / 4; ++q) {
      const float4 x0 = __ldg(c0 + q), x1 = __ldg(c1 + q);
      const float4 rv = *reinterpret_cast<const float4*>(res + 4 * q);
      float d;
      d = __fsub_rn(rv.x, x0.x); a0 = __fadd_rn(a0, __fmul_rn(d, d));
      d = __fsub_rn(rv.y, x0.y); a0 = __fadd_rn(a0, __fmul_rn(d, d));
      d = __fsub_rn(rv.z, x0.z); a0 = __fadd_rn(a0, __fmul_rn(d, d));
      d = __fsub_rn(rv.w, x0.w); a0 = __fadd_rn(a0, __fmul_rn(d, d));
      d = __fsub_rn(rv.x, x1.x); a1 = __fadd_rn(a1, __fmul_rn(d, d));
      d = __fsub_rn(rv.y, x1.y); a1 = __fadd_rn(a1, __fmul_rn(d, d));
      d = __fsub_rn(rv.z, x1.z); a1 = __fadd_rn(a1, __fmul_rn(d, d));
      d = __fsub_rn(rv.w, x1.w); a1 = __fadd_rn(a1, __fmul_rn(d, d));
    }
    // arg-min over (distance, code): this lane's two, then the warp
    float bd = a0;
    int bc = lane;
    if (a1 < bd) { bd = a1; bc = lane + 32; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, bd, o);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      if (od < bd || (od == bd && oc < bc)) { bd = od; bc = oc; }
    }
    if (lane == 0) {
      uint8_t* row = rows + static_cast<size_t>(r) * row_bytes;
      if (packed6) {
        // code p: bits 6p .. 6p+5 of the row, in byte 6p / 8 and, past bit 2 of it, the next
        const int bit = 6 * p, by = bit >> 3, sh = bit & 7;
        uint32_t w = row[by];
        if (sh > 2) w |= static_cast<uint32_t>(row[by + 1]) << 8;
        w = (w & ~(63u << sh)) | (static_cast<uint32_t>(bc) << sh);
        row[by] = static_cast<uint8_t>(w);
        if (sh > 2) row[by + 1] = static_cast<uint8_t>(w >> 8);
      } else {
        row[p] = static_cast<uint8_t>(bc);
      }
    }
    const float* chosen = cb + (static_cast<size_t>(r) * kWideCodes + bc) * kWideVDims;
    const float n0 = __fsub_rn(res[lane], __ldg(chosen + lane));
    const float n1 = __fsub_rn(res[lane + 32], __ldg(chosen + lane + 32));
    __syncwarp();                                                // every lane read res
    res[lane] = n0;
    res[lane + 32] = n1;
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_encode_append(const cvq_shape& s, const float* keys, const float* values,
                                 const float* key_cb, long long key_stride, const float* val_cb,
                                 long long val_stride, const int32_t* positions,
                                 uint8_t* key_codes, uint8_t* val_codes, cudaStream_t stream) {
  if (s.group_dim == kWideGroupDim) {
    const int n_units = s.batch * s.n_kv_heads * 2 * kWideGroups;
    const unsigned blocks = static_cast<unsigned>((n_units + kWideEncWarps - 1) / kWideEncWarps);
    encode_wide_kernel<<<blocks, 32 * kWideEncWarps, 0, stream>>>(
        keys, values, key_cb, key_stride, val_cb, val_stride, positions, key_codes, val_codes,
        s.R, s.n_kv_heads, s.t_cap, n_units, s.code_bits == 6);
    return cudaGetLastError();
  }
  // units = B * Hkv * 2 * 16, a multiple of kEncWarps
  const unsigned blocks = static_cast<unsigned>(s.batch) * s.n_kv_heads * 32 / kEncWarps;
  encode_kernel<<<blocks, 32 * kEncWarps, 0, stream>>>(keys, values, key_cb, key_stride, val_cb,
                                                        val_stride, positions, key_codes, val_codes,
                                                        s.R, s.n_kv_heads, s.t_cap);
  return cudaGetLastError();
}

}  // namespace cvq
