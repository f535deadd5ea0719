// Split-T flash-decode over the uint8 code stream: the straightforward form.
//
// One CTA = (split, head, sequence); one thread = one token of a 256-token tile (on splits
// of at most 128 tokens: 4 threads = one token of a 64-token tile, see TPT below).
// Per token: gather the key codewords of every (group, round) from the table
// (global memory, L1/L2 cached), sum the rounds, rotate by the RoPE phase
// e^{i theta_j t} and project on the query head(s) -> score (in log2 units).
// Online softmax per tile; the weights are accumulated per value code in
// shared-memory bins (the CommVQ value reorder: softmax weights multiply the value
// codes before the value codebook multiply -- review page, "forward_implications",
// 4th item).  Epilogue: o = bins x val_cb.
//
// Table form (TABLE = true, NG = 1): key_tab is the P table of one query head and
// the projection is the real part, Re(e^{i theta t} sum_r P).
// GQA form (TABLE = false): key_tab is the key codebook of one KV head and the
// projection is onto the NG query heads of its group, Re(conj(q) e^{i theta t} c).
#include "common.cuh"

namespace cvq {

constexpr int kSimpleThreads = 256;

// Threads per token.  TPT = 1: one thread walks a token's 16 groups.  TPT = 4 (for splits of
// at most kShortSplit tokens): 4 consecutive lanes share a token, lane `part` taking groups
// 4 part .. 4 part + 3, and a 2-level shuffle adds their partial scores, so a short split
// keeps all 8 warps busy with a 4x shorter dependent chain per thread.
constexpr int kShortSplit = 128;

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

template <int NG, int R, bool TABLE, int TPT>
__global__ void __launch_bounds__(kSimpleThreads) decode_simple_kernel(const DecodeArgs a) {
  static_assert(TPT == 1 || TPT == 4, "threads per token");
  // warps per query head in the fused merge
  constexpr int kMergeW = (kSimpleThreads / 32) / NG >= 4 ? 4 : (kSimpleThreads / 32) / NG;
  constexpr int kTileTokens = kSimpleThreads / TPT;
  extern __shared__ float4 smem_f4[];
  float* bins = reinterpret_cast<float*>(smem_f4);                // [NG][16][R][256]
  __shared__ float qs[NG][kHeadDim];
  __shared__ float red[kSimpleThreads / 32][NG];
  __shared__ float tmax[NG];

  const int split = blockIdx.x;
  const int head = blockIdx.y;      // TABLE: query head; GQA: KV head
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int group = a.n_q_heads / a.n_kv_heads;
  const int h = TABLE ? head / group : head;     // KV head
  const int hq0 = TABLE ? head : head * NG;       // first query head handled

  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.t_cap ? a.t_cap : L);
  const int t_begin = split * a.split_tokens;
  const int t_end = min(t_begin + a.split_tokens, L);

  const size_t part_row = (static_cast<size_t>(b) * a.n_q_heads + hq0) * a.n_splits + split;
  if (t_begin >= t_end) {
    for (int i = tid; i < NG * kHeadDim; i += kSimpleThreads) {
      const int hh = i / kHeadDim;
      a.part_o[(part_row + static_cast<size_t>(hh) * a.n_splits) * kHeadDim + (i % kHeadDim)] = 0.f;
    }
    if (tid < NG) {
      a.part_m[part_row + static_cast<size_t>(tid) * a.n_splits] = -INFINITY;
      a.part_l[part_row + static_cast<size_t>(tid) * a.n_splits] = 0.f;
    }
    if constexpr (!TABLE) {   // the fused merge serves cvq_attend (GQA form) only
      if (a.counters != nullptr) merge_tail<kMergeW, 4 * kMergeW>(a, b, head, hq0, NG, a.n_splits);
    }
    return;
  }

  const float qscale = kLog2e * 0.08838834764831845f;   // log2(e) / sqrt(128)
  for (int i = tid; i < NG * kHeadDim; i += kSimpleThreads) {
    const int hh = i / kHeadDim, d = i % kHeadDim;
    float v;
    if (TABLE) {
      v = (d & 1) ? 0.f : qscale;
    } else {
      v = load_q(a.q, a.q_dtype, (static_cast<size_t>(b) * a.n_q_heads + hq0 + hh) * kHeadDim + d) * qscale;
    }
    qs[hh][d] = v;
  }
  for (int i = tid; i < NG * kGroups * R * kCodes / 4; i += kSimpleThreads)
    reinterpret_cast<float4*>(bins)[i] = make_float4(0.f, 0.f, 0.f, 0.f);

  const float* tab = TABLE ? a.key_tab + (static_cast<size_t>(b) * a.n_q_heads + head) * a.key_tab_stride
                           : a.key_tab + static_cast<size_t>(h) * a.key_tab_stride;
  const size_t code_row = (static_cast<size_t>(b) * a.n_kv_heads + h) * a.t_cap;
  const uint4* kcodes = reinterpret_cast<const uint4*>(a.key_codes) + code_row * R;
  const uint4* vcodes = reinterpret_cast<const uint4*>(a.val_codes) + code_row * R;

  float m_run[NG], l_run[NG];
#pragma unroll
  for (int hh = 0; hh < NG; ++hh) { m_run[hh] = -INFINITY; l_run[hh] = 0.f; }
  __syncthreads();

  const int part = tid % TPT;                   // TPT = 4: this lane's groups 4 part .. + 3
  for (int t0 = t_begin; t0 < t_end; t0 += kTileTokens) {
    const int t = t0 + tid / TPT;
    const bool valid = t < t_end;
    uint4 kc[R], vc[R];
    float s[NG];
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) s[hh] = -INFINITY;
    if (valid) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        kc[r] = __ldg(kcodes + static_cast<size_t>(t) * R + r);
        vc[r] = __ldg(vcodes + static_cast<size_t>(t) * R + r);
      }
#pragma unroll
      for (int hh = 0; hh < NG; ++hh) s[hh] = 0.f;
      uint32_t kword[R];                        // TPT = 4: the key code bytes of this lane's groups
#pragma unroll
      for (int r = 0; r < R; ++r) kword[r] = word_of(kc[r], part);
#pragma unroll 4
      for (int gi = 0; gi < kGroups / TPT; ++gi) {
        const int G = TPT == 1 ? gi : 4 * part + gi;
        float kr[4] = {0.f, 0.f, 0.f, 0.f}, ki[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int c = TPT == 1 ? code_byte(kc[r], gi) : static_cast<int>((kword[r] >> (8 * gi)) & 255u);
          const float4* cw = reinterpret_cast<const float4*>(
              tab + ((static_cast<size_t>(G) * R + r) * kCodes + c) * kCodeword);
          const float4 lo = __ldg(cw), hi = __ldg(cw + 1);
          kr[0] += lo.x; ki[0] += lo.y; kr[1] += lo.z; ki[1] += lo.w;
          kr[2] += hi.x; ki[2] += hi.y; kr[3] += hi.z; ki[3] += hi.w;
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int j = 4 * G + p;
          const float2 ph = phase_at(a.phase.F[j], t);
          const float xr = ph.x * kr[p] - ph.y * ki[p];
          const float xi = ph.y * kr[p] + ph.x * ki[p];
#pragma unroll
          for (int hh = 0; hh < NG; ++hh) s[hh] += qs[hh][2 * j] * xr + qs[hh][2 * j + 1] * xi;
        }
      }
    }
    if constexpr (TPT > 1) {                    // add the partial scores of the token's lanes
#pragma unroll
      for (int o = 1; o < TPT; o <<= 1) {
#pragma unroll
        for (int hh = 0; hh < NG; ++hh) s[hh] += __shfl_xor_sync(0xffffffffu, s[hh], o);
      }
    }
    // tile max per head
    const int warp = tid / 32, lane = tid % 32;
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) {
      float v = s[hh];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0) red[warp][hh] = v;
    }
    __syncthreads();
    if (tid < NG) {
      float v = red[0][tid];
      for (int w = 1; w < kSimpleThreads / 32; ++w) v = fmaxf(v, red[w][tid]);
      tmax[tid] = v;
    }
    __syncthreads();
    bool rescaled = false;
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) {
      const float m_new = fmaxf(m_run[hh], tmax[hh]);
      if (m_new > m_run[hh]) {
        const float sc = exp2f(m_run[hh] - m_new);
        l_run[hh] *= sc;
        float* bh = bins + hh * kGroups * R * kCodes;
        for (int i = tid; i < kGroups * R * kCodes; i += kSimpleThreads) bh[i] *= sc;
        m_run[hh] = m_new;
        rescaled = true;
      }
    }
    if (rescaled) __syncthreads();     // uniform: every thread sees the same tmax
    if (valid) {
#pragma unroll
      for (int hh = 0; hh < NG; ++hh) {
        const float w = exp2f(s[hh] - m_run[hh]);
        if (part == 0) l_run[hh] += w;          // once per token
        float* bh = bins + hh * kGroups * R * kCodes;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t vword = word_of(vc[r], part);
#pragma unroll
          for (int gi = 0; gi < kGroups / TPT; ++gi) {
            const int G = TPT == 1 ? gi : 4 * part + gi;
            const int c = TPT == 1 ? code_byte(vc[r], gi) : static_cast<int>((vword >> (8 * gi)) & 255u);
            if (in_bounds(a.fault, (G * R + r) * kCodes + c, kGroups * R * kCodes))
              atomicAdd(bh + (G * R + r) * kCodes + c, w);
          }
        }
      }
    }
  }
  __syncthreads();
  // l: block sum per head
  {
    const int warp = tid / 32, lane = tid % 32;
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) {
      float v = l_run[hh];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][hh] = v;
    }
    __syncthreads();
    if (tid < NG) {
      float v = 0.f;
      for (int w = 0; w < kSimpleThreads / 32; ++w) v += red[w][tid];
      a.part_l[part_row + static_cast<size_t>(tid) * a.n_splits] = v;
      a.part_m[part_row + static_cast<size_t>(tid) * a.n_splits] = m_run[tid] * kLn2;
    }
  }
  // epilogue: o[hh][8G + d] = sum_{r, c} bins[hh][G][r][c] * val_cb[G][r][c][d].
  // Thread = (group G, code lane ch): it sums the codes ch, ch + 16, ... of its group over
  // all 8 dims of the group (two 16-byte loads per code, many in flight), then the 16 code
  // lanes of a half-warp reduce-scatter their 8 sums so that each dim ends on one lane.
  {
    static_assert(kGroups * 16 == kSimpleThreads, "one thread per (group, code lane)");
    constexpr int kSteps = R * kCodes / 16;
    const int G = tid >> 4, ch = tid & 15;
    const float4* vcb = reinterpret_cast<const float4*>(a.val_cb + static_cast<size_t>(h) * a.val_cb_stride) +
                        static_cast<size_t>(G) * R * kCodes * 2;
    float acc[NG][8];
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) {
#pragma unroll
      for (int d = 0; d < 8; ++d) acc[hh][d] = 0.f;
    }
    // odd groups start one step later: the two half-warps then read opposite bank halves
    const int k0 = G & 1;
#pragma unroll 8
    for (int k = 0; k < kSteps; ++k) {
      const int kk = (k + k0 == kSteps) ? 0 : k + k0;
      const int rc = kk * 16 + ch;                      // r * 256 + c
      const float4 v0 = __ldg(vcb + rc * 2), v1 = __ldg(vcb + rc * 2 + 1);
#pragma unroll
      for (int hh = 0; hh < NG; ++hh) {
        const float w = bins[(hh * kGroups + G) * R * kCodes + rc];
        acc[hh][0] = fmaf(w, v0.x, acc[hh][0]); acc[hh][1] = fmaf(w, v0.y, acc[hh][1]);
        acc[hh][2] = fmaf(w, v0.z, acc[hh][2]); acc[hh][3] = fmaf(w, v0.w, acc[hh][3]);
        acc[hh][4] = fmaf(w, v1.x, acc[hh][4]); acc[hh][5] = fmaf(w, v1.y, acc[hh][5]);
        acc[hh][6] = fmaf(w, v1.z, acc[hh][6]); acc[hh][7] = fmaf(w, v1.w, acc[hh][7]);
      }
    }
    const bool b3 = ch & 8, b2 = ch & 4, b1 = ch & 2;
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) {
      float* v = acc[hh];
#pragma unroll
      for (int i = 0; i < 4; ++i) {      // lanes differing in bit 3: keep dims 4 b3 + i
        const float send = b3 ? v[i] : v[i + 4];
        v[i] = (b3 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {      // bit 2: keep dims 4 b3 + 2 b2 + i
        const float send = b2 ? v[i] : v[i + 2];
        v[i] = (b2 ? v[i + 2] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      {                                  // bit 1: keep dim 4 b3 + 2 b2 + b1
        const float send = b1 ? v[0] : v[1];
        v[0] = (b1 ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, send, 2);
      }
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
      if ((ch & 1) == 0) {
        const int dim = G * kVDims + (ch >> 1);         // ch >> 1 = 4 b3 + 2 b2 + b1
        a.part_o[(part_row + static_cast<size_t>(hh) * a.n_splits) * kHeadDim + dim] = v[0];
      }
    }
  }
  if constexpr (!TABLE) {
    if (a.counters != nullptr) merge_tail<kMergeW, 4 * kMergeW>(a, b, head, hq0, NG, a.n_splits);
  }
}

template <int NG, int R, bool TABLE>
static cudaError_t launch_simple(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(NG) * kGroups * R * kCodes * sizeof(float);
  const bool short_split = a.split_tokens <= kShortSplit;
  auto k = short_split ? decode_simple_kernel<NG, R, TABLE, 4> : decode_simple_kernel<NG, R, TABLE, 1>;
  static PerDeviceFlag smem_set_short, smem_set_long;
  cudaError_t e = set_smem_limit_once(short_split ? smem_set_short : smem_set_long, k, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_splits, TABLE ? s.n_q_heads : s.n_kv_heads, s.batch);
  k<<<grid, kSimpleThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_table(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream) {
  return s.R == 1 ? launch_simple<1, 1, true>(s, a, stream) : launch_simple<1, 2, true>(s, a, stream);
}

cudaError_t launch_decode_gqa(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream) {
  const int g = s.n_q_heads / s.n_kv_heads;
  switch (g * 10 + s.R) {
    case 11: return launch_simple<1, 1, false>(s, a, stream);
    case 12: return launch_simple<1, 2, false>(s, a, stream);
    case 21: return launch_simple<2, 1, false>(s, a, stream);
    case 22: return launch_simple<2, 2, false>(s, a, stream);
    case 41:
    case 42: return launch_decode_gqa4(s, a, stream);
    case 81: return launch_simple<8, 1, false>(s, a, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace cvq
