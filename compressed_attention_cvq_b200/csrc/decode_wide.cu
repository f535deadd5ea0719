// Split-T flash-decode over the code stream with the paper's own parameterization:
// 64-entry codebooks over groups of 64 scalars (32 RoPE pairs share one index per round),
// R rounds (R = 11 gives 1.03 bits per scalar, R = 21 gives 1.97), 4 query heads per KV
// head (CommVQ summary page, "Key results" and "Limitations"; review page
// "key_machinery").
//
// Work unit: one (sequence b, KV head h, split s), handled by a cluster of
// C = 2 * ceil(R / 11) CTAs.  CTA rank rho owns group G = rho % 2 and the round slice
// rs = rho / 2, i.e. rounds [rs * RC, rs * RC + rc) with RC = ceil(R / ceil(R / 11)).
// Its shared memory holds those rounds' key codewords (rc x 16 KiB) and their value bins.
//
// Per token (8 lanes, each 4 of the group's 32 pairs):
//   1. sum the rc key codewords of the token's codes;
//   2. rotate each pair by its RoPE phase e^{i theta_j t} (the codeword commutes with the
//      rotation) and project on the 4 query heads: this CTA's share of the 4 scores;
//   3. reduce the share over the token's 8 lanes.
// Once per 256-token tile the C CTAs exchange their shares through distributed shared
// memory and add them in rank order, so every CTA holds bit-identical scores and runs the
// same online softmax (a reference max per head, raised only when a tile's max exceeds it
// by more than 8 in log2 units).  Each CTA then adds the weights to the value bins of its
// own rounds.  Epilogue: o = bins x value codewords (staged over the key-codeword region);
// the round slices of one group add their outputs through distributed shared memory.
//
// Layouts in shared memory (32 banks x 4 bytes):
//   key / value codewords: [rc][64 codes][16 chunks of 16 bytes] -- the global layout of
//     the group's rounds, so each round arrives by one TMA bulk copy; lane k of a token
//     reads chunks k and 8 + k, so the 8 lanes of a quarter-warp read 128 contiguous bytes;
//   bins: float c * 64 + 4 r + head; a warp's 8 tokens bin 8 different rounds at each
//     atomic step (the token's slot in the warp rotates its round order), so the 32 lanes
//     of an atomic hit 32 different banks whatever the codes;
//   codes: [buffer][key | value][rc][256 tokens] bytes, copied with cp.async from the
//     planar global layout [B, Hkv, 2, R, t_cap] while the previous tile computes, then
//     transposed once per tile to [key | value][256 tokens][16 bytes] so a token's rc codes
//     come in one 16-byte load; a token's value bytes are stored rotated to the round order
//     of its bin updates (its token slot's starting round first), so the update loop reads
//     byte i at a position fixed at compile time.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace cvq {

namespace {

constexpr int kWHeads = 4;
constexpr int kWTile = 256;
constexpr int kWThreads = 512;
constexpr int kWWarps = kWThreads / 32;
constexpr int kWSlots = kWWarps * 4;              // tokens per step
constexpr int kWSteps = kWTile / kWSlots;         // steps per tile
constexpr int kWChunks = kWidePairs * 2 / 4;      // 16-byte chunks per codeword (16)
constexpr int kBinStride = 64;                     // floats per code: 4 r + head, r < 11
constexpr float kWSlack = 8.0f;
constexpr int kRC = kWideRoundsPerCta;

constexpr size_t kCwBytes = sizeof(float4) * kRC * kWideCodes * kWChunks;   // 180,224
constexpr size_t kBinBytes = sizeof(float) * kWideCodes * kBinStride;      //  16,384
static_assert(4 * kRC <= kBinStride, "bins of one code");
constexpr size_t kXchgBytes = sizeof(float) * 2 * kWTile * kWHeads;         //   8,192
constexpr size_t kCodeBytes = 2 * 2 * kRC * kWTile;                         //  11,264
constexpr size_t kTCodeBytes = 2 * kWTile * 16;                              //   8,192
constexpr size_t kRedBytes = sizeof(float) * (2 * kWWarps * kWHeads + 4 * kWHeads);
constexpr size_t kWSmem = kCwBytes + kBinBytes + kXchgBytes + kCodeBytes + kTCodeBytes + kRedBytes;
static_assert(kWSteps * kWSlots == kWTile, "tile must be a whole number of steps");
static_assert(kWSmem <= 227 * 1024, "shared memory per CTA");
// the reduction region holds red_m, red_l, mref_s, l_s, 16 unused bytes and, in its last 16
// bytes, the 8-byte mbarrier of the codebook copies
static_assert(kRedBytes >= sizeof(float) * (2 * kWWarps * kWHeads + 3 * kWHeads) + 8, "mbarrier room");
static_assert((kCwBytes + kBinBytes + kXchgBytes + kCodeBytes + kTCodeBytes +
               sizeof(float) * (2 * kWWarps * kWHeads + 3 * kWHeads)) % 8 == 0, "mbarrier alignment");

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}

// Copy rc rounds x 64 codewords of one group (a contiguous run of rc * 4096 floats) with
// one TMA bulk copy per round, issued by lanes 0 .. rc-1 of warp 0 after lane 0 set the
// transaction count.
__device__ __forceinline__ void stage_codebook(float4* dst, const float* src, int rc, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  constexpr unsigned kRound = static_cast<unsigned>(sizeof(float4)) * kWideCodes * kWChunks;
  if (lane == 0) mbar_expect_tx(bar, kRound * rc);
  __syncwarp();
  if (lane < rc) bulk_load(dst + lane * kWideCodes * kWChunks, src + lane * kWideCodes * 4 * kWChunks, kRound, bar);
}

// One CTA's work.  kRounds > 0: the CTA's round slice holds exactly kRounds rounds, so the
// round loops run without a per-round bound check; 0: the slice size is computed at run time.
template <int kRounds>
__device__ __forceinline__ void wide_body(const DecodeArgs& a, int R) {
  extern __shared__ __align__(128) float4 smem4[];
  float4* cw_s = smem4;                                                       // codewords
  float* bins = reinterpret_cast<float*>(smem4 + kRC * kWideCodes * kWChunks);
  float* xchg = bins + kWideCodes * kBinStride;                               // [2][256][4]
  uint8_t* code_s = reinterpret_cast<uint8_t*>(xchg + 2 * kWTile * kWHeads);  // [2][2][rc][256]
  uint8_t* tcode = code_s + kCodeBytes;                                       // [2][256][16]
  float* red_m = reinterpret_cast<float*>(tcode + kTCodeBytes);              // [16][4]
  float* red_l = red_m + kWWarps * kWHeads;                                   // [16][4]
  float* mref_s = red_l + kWWarps * kWHeads;                                  // [4]
  float* l_s = mref_s + kWHeads;                                              // [4]
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(l_s + 2 * kWHeads);         // codebook copies

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rho = static_cast<int>(cluster.block_rank());
  const int G = rho & 1, rs = rho >> 1;
  const int n_slices = C >> 1;
  const int RCeil = (R + n_slices - 1) / n_slices;
  const int r0 = rs * RCeil;
  const int rc = kRounds > 0 ? kRounds : min(R, r0 + RCeil) - r0;

  const int split = blockIdx.x / C;
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tau = lane >> 3, k = lane & 7;
  const int hq0 = h * kWHeads;

  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.t_cap ? a.t_cap : L);
  const int t_begin = split * a.split_tokens;
  const int t_end = min(t_begin + a.split_tokens, L);
  const size_t part_row = (static_cast<size_t>(b) * a.n_q_heads + hq0) * a.n_splits + split;

  if (t_begin >= t_end) {   // every CTA of the cluster takes this branch
    if (rs == 0) {
      for (int i = tid; i < kWHeads * kWideVDims; i += kWThreads) {
        const int hh = i / kWideVDims, d = i % kWideVDims;
        a.part_o[(part_row + static_cast<size_t>(hh) * a.n_splits) * kHeadDim + G * kWideVDims + d] = 0.f;
      }
    }
    if (rho == 0 && tid < kWHeads) {
      a.part_m[part_row + static_cast<size_t>(tid) * a.n_splits] = -INFINITY;
      a.part_l[part_row + static_cast<size_t>(tid) * a.n_splits] = 0.f;
    }
    if (a.counters != nullptr) merge_tail(a, b, h, hq0, kWHeads, C * a.n_splits);
    return;
  }

  // planar codes: row (b, h, G, r) of t_cap bytes
  const size_t code_row0 = ((static_cast<size_t>(b) * a.n_kv_heads + h) * kWideGroups + G) * R + r0;
  // a code row holds t_cap bytes, or 3 t_cap / 4 packed (t_cap and every tile start a
  // multiple of 64, so a tile's packed bytes start on a 16-byte boundary); the tile's
  // 16-byte chunks that hold tokens before t_end are copied, never past the row's end
  const bool packed6 = a.code_bits == 6;
  const size_t row_bytes = packed6 ? static_cast<size_t>(a.t_cap) / 4 * 3 : static_cast<size_t>(a.t_cap);
  constexpr int kChunksPerRow = kWTile / 16;           // unpacked; packed uses 3/4 of them
  auto stage_codes = [&](int t_tile, int buf) {
    const int n = 2 * rc * kChunksPerRow;
    const size_t tile_byte = packed6 ? static_cast<size_t>(t_tile) / 4 * 3 : static_cast<size_t>(t_tile);
    const int need = packed6 ? ((t_end - t_tile) * 3 + 3) / 4 : (t_end - t_tile);   // bytes with tokens < t_end
    for (int i = tid; i < n; i += kWThreads) {
      const int kind = i / (rc * kChunksPerRow);
      const int r = (i / kChunksPerRow) % rc;
      const int q16 = i % kChunksPerRow;
      if (16 * q16 < need && in_bounds(a.fault, tile_byte + 16 * q16 + 15, row_bytes)) {
        const uint8_t* src = (kind ? a.val_codes : a.key_codes) + (code_row0 + r) * row_bytes + tile_byte + 16 * q16;
        cp_async16(code_s + ((buf * 2 + kind) * kRC + r) * kWTile + 16 * q16, src);
      }
    }
  };

  const float* kcb = a.key_tab + h * a.key_tab_stride +
                     (static_cast<size_t>(G) * R + r0) * kWideCodes * 2 * kWidePairs;
  const float* vcb = a.val_cb + h * a.val_cb_stride +
                     (static_cast<size_t>(G) * R + r0) * kWideCodes * kWideVDims;
  if (tid == 0) mbar_init(tma_bar, 1);
  if (warp == 0) stage_codebook(cw_s, kcb, rc, tma_bar);
  stage_codes(t_begin, 0);
  cp_async_commit();
  for (int i = tid; i < kWideCodes * kBinStride / 4; i += kWThreads)
    reinterpret_cast<float4*>(bins)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  // softmax state of head tid & 3, held by every thread: the reference max (the same in
  // every thread of the CTA) and this thread's share of l
  float m_ref = -INFINITY, l_acc = 0.f;

  // this lane's 4 pairs: local pairs 2k, 2k+1 (chunk k) and 2k+16, 2k+17 (chunk 8+k)
  int jp[4];
  jp[0] = G * kWidePairs + 2 * k;
  jp[1] = jp[0] + 1;
  jp[2] = jp[0] + 16;
  jp[3] = jp[0] + 17;
  unsigned long long F[4];
  float2 mul[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    F[p] = a.phase.F[jp[p]];
    mul[p] = phase_at(F[p], kWSlots);
  }
  // queries, scaled to log2 units; slot j holds head (k ^ j) & 3 (select-free reduction)
  const float qscale = kLog2e * 0.08838834764831845f;
  float2 qv[kWHeads][4];                 // (real, imaginary) of pair p for head slot j
#pragma unroll
  for (int j = 0; j < kWHeads; ++j) {
    const int hh = (k ^ j) & 3;
    const size_t qrow = (static_cast<size_t>(b) * a.n_q_heads + hq0 + hh) * kHeadDim;
#pragma unroll
    for (int p = 0; p < 4; ++p)
      qv[j][p] = make_float2(load_q(a.q, a.q_dtype, qrow + 2 * jp[p]) * qscale,
                             load_q(a.q, a.q_dtype, qrow + 2 * jp[p] + 1) * qscale);
  }

  const int n_tiles = (t_end - t_begin + kWTile - 1) / kWTile;
  const int tt0 = warp * 4 + tau;            // this lane's token slot in step 0
  for (int it = 0; it < n_tiles; ++it) {
    const int t_tile = t_begin + it * kWTile;
    const int buf = it & 1;
    cp_async_wait_all();
    __syncthreads();                          // codes of this tile landed
    // the key codewords (phase 0 of the barrier); a copy that never lands is reported in
    // the fault word and the kernel runs on, so that every CTA still meets every barrier
    if (it == 0 && !mbar_wait(tma_bar, 0) && tid == 0) atomicOr(a.fault, kFaultCopyTimeout);
    if (it + 1 < n_tiles) stage_codes(t_tile + kWTile, buf ^ 1);
    cp_async_commit();
    // token-major copy of this tile's codes: 16 bytes per (key | value, token), byte r =
    // round r, so one 16-byte load gives a token all its codes
    {
      const int kind = tid >> 8, t = tid & 255;
      const uint8_t* src = code_s + (buf * 2 + kind) * kRC * kWTile + t;
      uint32_t wv[4] = {0u, 0u, 0u, 0u};
      const uint8_t* srow = code_s + (buf * 2 + kind) * kRC * kWTile;     // packed rows
#pragma unroll
      for (int r = 0; r < kRC; ++r)
        if (r < rc) {
          const uint32_t c = packed6 ? static_cast<uint32_t>(packed6_code(srow + r * kWTile, t))
                                     : static_cast<uint32_t>(src[r * kWTile]);
          wv[r >> 2] |= c << (8 * (r & 3));
        }
      if (kind == 1) {
        // value codes in the order the token's bin updates take them: byte i = round
        // (rf + i) mod rc, rf = the round its token slot starts at (token t & 7 mod rc)
        const int rf = (t & 7) % rc;
        const unsigned __int128 v = (static_cast<unsigned __int128>(wv[2]) << 64) |
                                    (static_cast<unsigned __int128>(wv[1]) << 32) | wv[0];
        const unsigned __int128 mask = (static_cast<unsigned __int128>(1) << (8 * rc)) - 1;
        const unsigned __int128 rot =
            rf == 0 ? v : (((v >> (8 * rf)) | (v << (8 * (rc - rf)))) & mask);
        wv[0] = static_cast<uint32_t>(rot);
        wv[1] = static_cast<uint32_t>(rot >> 32);
        wv[2] = static_cast<uint32_t>(rot >> 64);
      }
      *reinterpret_cast<uint4*>(tcode + (kind * kWTile + t) * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
    __syncthreads();
    float* xo = xchg + buf * kWTile * kWHeads;

    // ---- this CTA's share of every token's 4 scores ----
    float2 ph[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) ph[p] = phase_at(F[p], t_tile + tt0);
    // four steps unrolled: the next token's codeword loads are issued while the previous
    // token's rotation, projection and shuffle reduction complete
#pragma unroll 4
    for (int step = 0; step < kWSteps; ++step) {
      const int tt = step * kWSlots + tt0;
      float2 acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
      if (t_tile + tt < t_end) {
        const uint4 kc4 = *reinterpret_cast<const uint4*>(tcode + tt * 16);
        const uint32_t kcw[4] = {kc4.x, kc4.y, kc4.z, kc4.w};
#pragma unroll
        for (int r = 0; r < kRC; ++r) {
          if (r < rc) {
            const int c = (kcw[r >> 2] >> (8 * (r & 3))) & (kWideCodes - 1);
            const float4* cwp = cw_s + (r * kWideCodes + c) * kWChunks;
            const float4 x = cwp[k], y = cwp[8 + k];
            acc[0] = __fadd2_rn(acc[0], make_float2(x.x, x.y));
            acc[1] = __fadd2_rn(acc[1], make_float2(x.z, x.w));
            acc[2] = __fadd2_rn(acc[2], make_float2(y.x, y.y));
            acc[3] = __fadd2_rn(acc[3], make_float2(y.z, y.w));
          }
        }
      }
      // rotate each pair, project on the 4 heads with packed (real, imaginary) FMAs
      float2 P2[kWHeads];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float xr = acc[p].x, xi = acc[p].y;
        const float2 z = make_float2(fmaf(ph[p].x, xr, -ph[p].y * xi), fmaf(ph[p].x, xi, ph[p].y * xr));
#pragma unroll
        for (int j = 0; j < kWHeads; ++j) P2[j] = p == 0 ? __fmul2_rn(qv[j][p], z) : __ffma2_rn(qv[j][p], z, P2[j]);
      }
      float P[kWHeads];
#pragma unroll
      for (int j = 0; j < kWHeads; ++j) P[j] = P2[j].x + P2[j].y;
      // sum over the token's 8 lanes; lane k ends with head k & 3
      const float s0 = P[0] + __shfl_xor_sync(0xffffffffu, P[2], 2);
      const float s1 = P[1] + __shfl_xor_sync(0xffffffffu, P[3], 2);
      float v = s0 + __shfl_xor_sync(0xffffffffu, s1, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      if (k < kWHeads) xo[tt * kWHeads + k] = v;
#pragma unroll
      for (int p = 0; p < 4; ++p) ph[p] = cmul(ph[p], mul[p]);
    }

    // ---- exchange: every CTA sums the C shares in rank order ----
    cluster_sync_all();
    const int hh = tid & 3;
    const int tA = tid >> 2, tB = tA + kWTile / 2;
    float sA = 0.f, sB = 0.f;
    for (int q = 0; q < C; ++q) {
      const float* px = cluster.map_shared_rank(xo, q);
      if (in_bounds(a.fault, tB * kWHeads + hh, kWTile * kWHeads)) {
        sA += px[tA * kWHeads + hh];
        sB += px[tB * kWHeads + hh];
      }
    }
    if (t_tile + tA >= t_end) sA = -INFINITY;
    if (t_tile + tB >= t_end) sB = -INFINITY;

    // ---- online softmax with a lagging reference max ----
    float mx = fmaxf(sA, sB);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (lane < kWHeads) red_m[warp * kWHeads + lane] = mx;
    __syncthreads();
    // every warp reduces the 16 warps' maxima itself (entry w * 4 + head): lane l takes
    // entries l and l + 32, then the lanes of its head; every thread ends with the same
    // tile max of head hh, so the decisions below are the same in every warp
    float tm = fmaxf(red_m[lane], red_m[lane + 32]);
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 4));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 8));
    tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
    const bool raise = tm > m_ref + kWSlack;
    if (__any_sync(0xffffffffu, raise)) {
      const float m_new = raise ? tm : m_ref;
      const float f = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - m_new);
      const bool rescale = __any_sync(0xffffffffu, m_ref != -INFINITY);
      l_acc *= f;
      m_ref = m_new;
      if (rescale) {   // every earlier atomic was issued before this tile's barriers
        const float f0 = __shfl_sync(0xffffffffu, f, 0), f1 = __shfl_sync(0xffffffffu, f, 1);
        const float f2 = __shfl_sync(0xffffffffu, f, 2), f3 = __shfl_sync(0xffffffffu, f, 3);
        for (int i = tid; i < kWideCodes * kBinStride; i += kWThreads) {
          const int e = i & 3;
          bins[i] *= e == 0 ? f0 : (e == 1 ? f1 : (e == 2 ? f2 : f3));
        }
        __syncthreads();
      }
    }
    const float wA = exp2f(sA - m_ref), wB = exp2f(sB - m_ref);
    l_acc += wA + wB;
    // value reorder: the weight goes to the bin of the token's value code, per own round
    // token slot j of the warp starts at round j (mod rc), so each atomic instruction's 8
    // tokens bin 8 different rounds
    const int r_first = (lane >> 2) % rc;
    auto bin_token = [&](int tt, float wt) {
      const uint4 v4 = *reinterpret_cast<const uint4*>(tcode + (kWTile + tt) * 16);
      int r = r_first;
#pragma unroll
      for (int i = 0; i < kRC; ++i) {
        if (i < rc) {
          // byte i holds round r = (r_first + i) mod rc (rotated in the transpose)
          const uint32_t wd = i < 4 ? v4.x : (i < 8 ? v4.y : v4.z);
          const int c = (wd >> (8 * (i & 3))) & (kWideCodes - 1);
          if (in_bounds(a.fault, c * kBinStride + 4 * r + hh, kWideCodes * kBinStride))
            atomicAdd(&bins[c * kBinStride + 4 * r + hh], wt);
          r = (r + 1 == rc) ? 0 : r + 1;
        }
      }
    };
    if (wA > 0.f) bin_token(tA, wA);
    if (wB > 0.f) bin_token(tB, wB);
  }
  // l per head: over the warp's lanes of the head, then over the 16 warps
  l_acc += __shfl_xor_sync(0xffffffffu, l_acc, 4);
  l_acc += __shfl_xor_sync(0xffffffffu, l_acc, 8);
  l_acc += __shfl_xor_sync(0xffffffffu, l_acc, 16);
  if (lane < kWHeads) red_l[warp * kWHeads + lane] = l_acc;
  __syncthreads();
  if (tid < kWHeads) {
    float l = 0.f;
    for (int w = 0; w < kWWarps; ++w) l += red_l[w * kWHeads + tid];
    l_s[tid] = l;
    mref_s[tid] = m_ref;                   // thread tid < 4: head tid
  }

  // ---- epilogue: o = bins x value codewords of the own rounds ----
  // (every read of the key codewords happened before the barrier above; the fence orders
  // them before the TMA writes)
  if (warp == 0) {
    fence_proxy_async_smem();
    stage_codebook(cw_s, vcb, rc, tma_bar);
  }
  if (!mbar_wait(tma_bar, 1) && tid == 0) atomicOr(a.fault, kFaultCopyTimeout);
  const float* cv = reinterpret_cast<const float*>(cw_s);
  const int eh = (tid >> 6) & 3, ed = tid & 63, half = tid >> 8;
  float o = 0.f;
  for (int r = 0; r < rc; ++r) {
    const float* br = bins + 4 * r + eh;
    const float* vr = cv + static_cast<size_t>(r) * kWideCodes * kWideVDims + ed;
#pragma unroll 8
    for (int c = half * 32; c < half * 32 + 32; ++c) o = fmaf(br[c * kBinStride], vr[c * kWideVDims], o);
  }
  // the xchg buffer the last tile did not use: no peer reads it any more
  float* ored = xchg + (n_tiles & 1) * kWTile * kWHeads;   // [256] halves, then [256] slice
  float* oslice = ored + kWHeads * kWideVDims;
  if (half) ored[eh * kWideVDims + ed] = o;
  __syncthreads();
  if (!half) {
    o += ored[eh * kWideVDims + ed];
    if (rs == 1) oslice[eh * kWideVDims + ed] = o;
  }
  cluster_sync_all();          // slices written; peers are done reading this CTA's xchg
  if (!half && rs == 0) {
    if (n_slices == 2) o += cluster.map_shared_rank(oslice, rho + 2)[eh * kWideVDims + ed];
    a.part_o[(part_row + static_cast<size_t>(eh) * a.n_splits) * kHeadDim + G * kWideVDims + ed] = o;
  }
  if (rho == 0 && tid < kWHeads) {
    a.part_m[part_row + static_cast<size_t>(tid) * a.n_splits] = mref_s[tid] * kLn2;
    a.part_l[part_row + static_cast<size_t>(tid) * a.n_splits] = l_s[tid];
  }
  cluster_sync_all();          // keep oslice alive until the peer has read it
  if (a.counters != nullptr) merge_tail(a, b, h, hq0, kWHeads, C * a.n_splits);
}

// kFirst / kRest: the rounds of the first round slice / of the others, known when the kernel
// is compiled (0: computed at run time).  Every CTA of a cluster meets the same barriers
// whichever body it runs.
template <int kFirst, int kRest>
__global__ void __launch_bounds__(kWThreads, 1) decode_wide_kernel(const __grid_constant__ DecodeArgs a, int R) {
  if (kFirst == kRest || (cg::this_cluster().block_rank() >> 1) == 0) {
    wide_body<kFirst>(a, R);
  } else {
    wide_body<kRest>(a, R);
  }
}

template <int kFirst, int kRest>
cudaError_t launch_wide(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream) {
  const int C = wide_cluster_size(s.R);
  static PerDeviceFlag smem_set;
  cudaError_t e = set_smem_limit_once(smem_set, decode_wide_kernel<kFirst, kRest>, kWSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.n_splits * C), s.n_kv_heads, s.batch);
  cfg.blockDim = dim3(kWThreads);
  cfg.dynamicSmemBytes = kWSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_wide_kernel<kFirst, kRest>, a, s.R);
}

}  // namespace

cudaError_t launch_decode_wide(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream) {
  // R = 11 or 22: every round slice is 11 rounds; R = 21: slices of 11 and 10 rounds
  if (s.R % kRC == 0) return launch_wide<kRC, kRC>(s, a, stream);
  if (s.R == 2 * kRC - 1) return launch_wide<kRC, kRC - 1>(s, a, stream);
  return launch_wide<0, 0>(s, a, stream);
}

}  // namespace cvq
