// Split-T flash-decode over the uint8 code stream, GQA form, for groups of 4 query
// heads per KV head (the LLaMA-3.1-8B shape).
//
// Work unit: one (sequence b, KV head h, split s), handled by a cluster of two CTAs.
// CTA rank g of the pair owns key/value groups 8g .. 8g+7, so its shared memory holds
// half of each codebook (64R KiB of key codewords, 32R KiB of value bins) and both
// residual depths fit on chip.
//
// Per token and KV head (CommVQ review page, "key_machinery" and "forward_implications"):
//   1. gather sum_r c[G, r, key_code] for the CTA's 8 groups (8 lanes per token, one
//      group = 4 RoPE pairs per lane);
//   2. rotate by the RoPE phase e^{i theta_j t} -- the codeword commutes with the rotation,
//      so this equals rotating the key -- and project on the 4 query heads;
//   3. reduce the partial scores over the token's 8 lanes, exchange them with the peer
//      CTA through distributed shared memory and add: the score of every head;
//   4. online softmax with a reference max per head that is raised only when a tile's
//      max exceeds it by more than 8 (log2 units), so the bins are rescaled rarely;
//   5. add the weight of every head to the bin of the token's value code, per group and
//      round (the value reorder: weights multiply value codes before the codebook);
//   6. epilogue: o = bins x value codebook for the CTA's 64 output dims.
//
// Shared-memory layouts, chosen for conflict-free access (32 banks x 4 bytes):
//   key / value codewords: [r][c][G_local][8 floats], staged by TMA (8 tiled copies of
//     32 codes per round, 32-byte rows); the lanes of groups 0-3 read the lower 16-byte
//     half of their codeword first and those of groups 4-7 the upper half, so the 8 lanes
//     of a quarter-warp (one token, groups 0..7) hit 8 different bank groups;
//   bins: float ((r*256 + c)*4 + head)*8 + G_local; at every atomic step the 32 lanes
//     of a warp (4 tokens x 4 heads x 2 group halves, each token on a rotated group)
//     touch 32 different banks and never the same address.
//
// Tokens: kSlots = 4 per warp per step; slot sigma handles t_begin + sigma + kSlots*j.
// The phase of a lane's 4 pairs is re-seeded from the exact fixed-point turn at the start
// of every tile and advances by e^{i theta_j kSlots} per step within it (at most
// kSteps - 1 = 7 products at R = 1, 3 at R = 2, rounding error ~1e-7 each).  Each warp
// copies the code bytes of its own token slots for the next tile to shared memory with
// cp.async while the current tile computes, so the only barrier of a tile is the cluster
// barrier of the score exchange.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace cvq {

namespace {

constexpr int kHeads = 4;              // query heads per KV head
constexpr int kLocalGroups = 8;        // groups per CTA of the pair
constexpr int kTile = 256;             // tokens per tile (softmax / exchange period)
constexpr float kRescaleSlack = 8.0f;  // log2 units the reference max may lag behind

template <int R>
struct Cfg {
  static constexpr int kThreads = (R == 1) ? 256 : 512;
  static constexpr int kWarps = kThreads / 32;
  static constexpr int kSlots = kWarps * 4;                  // tokens per step
  static constexpr int kSteps = kTile / kSlots;              // steps per tile
  static constexpr int kMinBlocks = (R == 1) ? 2 : 1;
  static constexpr int kCodeChunks = R * kCodes * 2 * kLocalGroups;   // 16-byte chunks
  static constexpr int kBins = R * kCodes * kHeads * kLocalGroups;    // floats
  static constexpr int kXchg = 2 * kTile * kHeads;                    // floats (2 buffers)
  static constexpr int kCodeBytes = 2 * kTile * R * 16;               // 2 buffers x (key 8 B + val 8 B) x R
  static constexpr size_t kSmem = sizeof(float4) * kCodeChunks +
                                  sizeof(float) * (kBins + kXchg + kWarps * kHeads + 4 * kHeads) +
                                  kCodeBytes + 16 +   // + the TMA mbarrier
                                  sizeof(unsigned long long) * 4 * kLocalGroups;   // phase turns
  static_assert(kSteps * kSlots == kTile, "tile must be a whole number of steps");
};

__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// One CTA's half of a codebook (local groups 8 rank .. 8 rank + 7, every round and code)
// into the chunk layout of cw_s, by 8 R tiled TMA copies of 32 codes each, issued by lanes
// 0 .. 8R-1 of one warp after lane 0 set the transaction count.  Called by a whole warp.
template <int R>
__device__ __forceinline__ void stage_codebook_tma(float4* cw_s, const CUtensorMap* map, int rank, int head,
                                                   uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) mbar_expect_tx(bar, static_cast<unsigned>(sizeof(float4)) * R * kCodes * 2 * kLocalGroups);
  __syncwarp();
  if (lane < 8 * R) {
    const int rc = lane * kCodeBoxRows;                 // round * 256 + first code
    tma_load_4d(cw_s + rc * kLocalGroups * 2, map, 0, rank * kLocalGroups, rc, head, bar);
  }
}

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}

template <int R>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<R>::kThreads, Cfg<R>::kMinBlocks)
    decode_gqa4_kernel(const __grid_constant__ DecodeArgs a) {
  using C = Cfg<R>;
  extern __shared__ __align__(128) float4 smem4[];
  float4* cw_s = smem4;                                               // [R][256][8][2] chunks
  float* bins = reinterpret_cast<float*>(smem4 + C::kCodeChunks);     // [R][256][4][8]
  float* xchg = bins + C::kBins;                                      // [2][kTile][4]
  float* red = xchg + C::kXchg;                                       // [kWarps][4]
  float* fh = red + C::kWarps * kHeads;                               // [4] rescale factors
  int* mslot = reinterpret_cast<int*>(fh + kHeads);                   // [3][4] tile maxima (ord)
  uint8_t* code_s = reinterpret_cast<uint8_t*>(mslot + 3 * kHeads);   // [2][kTile][R][key 8 | val 8]
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(code_s + C::kCodeBytes);   // codebook copies
  // F_j of the CTA's 32 pairs (local group k: pairs 4 k .. 4 k + 3), read at every tile's
  // phase re-seed from shared memory instead of the parameter space
  unsigned long long* f_s = reinterpret_cast<unsigned long long*>(code_s + C::kCodeBytes + 16);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());           // which half of the groups
  const int split = blockIdx.x >> 1;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int tau = lane >> 3;               // token slot within the warp (0..3)
  const int k = lane & 7;                  // local group of the key side
  const int fk = k >> 2;                   // which codeword half this lane reads first
  const int hk = k & 3;                    // head whose score / weights this lane keeps
  const int gh = k >> 2;                   // which 4 local groups this lane bins
  const int sigma = warp * 4 + tau;        // token slot within the step
  const int hq0 = h * kHeads;

  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.t_cap ? a.t_cap : L);
  const int t_begin = split * a.split_tokens;
  const int t_end = min(t_begin + a.split_tokens, L);
  const size_t part_row = (static_cast<size_t>(b) * a.n_q_heads + hq0) * a.n_splits + split;
  // the last partial-state row this CTA writes lies inside the partial states
  const bool parts_ok = in_bounds(a.fault, part_row + static_cast<size_t>(kHeads - 1) * a.n_splits,
                                  static_cast<size_t>(a.batch) * a.n_q_heads * a.n_splits);

  if (t_begin >= t_end) {   // both CTAs of the pair take this branch together
    for (int i = tid; i < kHeads * 64 && parts_ok; i += C::kThreads) {
      const int hh = i >> 6, d = i & 63;
      a.part_o[(part_row + static_cast<size_t>(hh) * a.n_splits) * kHeadDim + rank * 64 + d] = 0.f;
    }
    if (rank == 0 && tid < kHeads && parts_ok) {
      a.part_m[part_row + static_cast<size_t>(tid) * a.n_splits] = -INFINITY;
      a.part_l[part_row + static_cast<size_t>(tid) * a.n_splits] = 0.f;
    }
    if (a.counters != nullptr) merge_tail(a, b, h, hq0, kHeads, 2 * a.n_splits);
    return;
  }

  const size_t code_row = (static_cast<size_t>(b) * a.n_kv_heads + h) * a.t_cap;
  // copy the code bytes of this CTA's 8 groups for one tile (key and value, every round)
  // each warp copies the code bytes of its own token slots (sigma = 4 warp + tau over the
  // tile's steps), so only the warp's own copies must land before it reads them: no
  // CTA-wide barrier per tile for the codes
  auto stage_codes = [&](int t_tile, int buf) {
    static_assert(C::kSteps * 4 * R == 32, "one (token, round) per lane and tile");
    {
      const int r = lane % R, slot = (lane / R) & 3, st = lane / (4 * R);
      const int tt = st * C::kSlots + warp * 4 + slot;
      const int t = t_tile + tt;
      if (t < t_end && in_bounds(a.fault, t, a.t_cap) &&
          in_bounds(a.fault, ((buf * kTile + tt) * R + r) * 16 + 15, C::kCodeBytes)) {
        const size_t off = (code_row + t) * (16 * R) + r * 16 + rank * 8;
        uint8_t* dst = code_s + ((buf * kTile + tt) * R + r) * 16;
        cp_async8(dst, a.key_codes + off);
        cp_async8(dst + 8, a.val_codes + off);
      }
    }
    cp_async_commit();
  };

  // ---- prologue: key codewords of this CTA's groups by TMA (tiled copies of groups
  // 8 rank .. 8 rank + 7, straight into the layout above), the first tile's codes by
  // cp.async ----
  if (warp == 0) {
    if (lane == 0) mbar_init(tma_bar, 1);
    stage_codebook_tma<R>(cw_s, &a.key_map, rank, a.key_tab_stride == 0 ? 0 : h, tma_bar);
  }
  stage_codes(t_begin, 0);
  for (int i = tid; i < C::kBins / 4; i += C::kThreads)
    reinterpret_cast<float4*>(bins)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (tid < 3 * kHeads) mslot[tid] = ord_of(-INFINITY);
  if (tid < 4 * kLocalGroups) f_s[tid] = a.phase.F[4 * rank * kLocalGroups + tid];

  // queries of the 4 heads for this lane's 4 pairs, scaled so that scores are in log2
  // units.  Slot j holds head (k ^ j) & 3: with this lane-dependent order the butterfly
  // that sums the partials over the token's 8 lanes needs no selects, and leaves head
  // k & 3 in lanes k and k ^ 4.
  // Lanes k = 4..7 read the upper half (pairs 2, 3) of their codeword first, so their
  // slots 0..3 hold pairs 2, 3, 0, 1 of the group (fk = 1); lanes 0..3 keep pairs 0..3.
  const float qscale = kLog2e * 0.08838834764831845f;
  const int G = rank * kLocalGroups + k;
  float2 qv[kHeads][4];
#pragma unroll
  for (int j = 0; j < kHeads; ++j) {
    const int hh = (k ^ j) & 3;
    const size_t qb = (static_cast<size_t>(b) * a.n_q_heads + hq0 + hh) * kHeadDim + 8 * G;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int pp = p ^ (2 * fk);                     // slot p holds pair 4 G + pp
      qv[j][p] = make_float2(load_q(a.q, a.q_dtype, qb + 2 * pp) * qscale,
                             load_q(a.q, a.q_dtype, qb + 2 * pp + 1) * qscale);
    }
  }
  // phase of the lane's pairs: re-seeded from the exact turn at the first token of every
  // tile, advanced by e^{i theta kSlots} per step within the tile
  float2 ph[4], adv[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) adv[p] = phase_at(a.phase.F[4 * G + (p ^ (2 * fk))], C::kSlots);
  float* peer_xchg = cluster.map_shared_rank(xchg, rank ^ 1);

  float m_ref = -INFINITY;      // reference max (log2 units) of head hk; equal in all lanes
  float l_acc = 0.f;            // this lane's share of sum_t w for head hk

  cp_async_wait_all();
  cluster.sync();               // bins and the first codes ready in both CTAs
  // the codewords (phase 0 of the barrier); a copy that never lands is reported in the
  // fault word and the kernel runs on, so that every CTA still meets every barrier
  if (!mbar_wait(tma_bar, 0) && tid == 0) atomicOr(a.fault, kFaultCopyTimeout);

  // per-lane float offsets into the bins: step i of a token's atomics adds to local group
  // 4 gh + ((i + tau) & 3) of head hk
  int bin_off[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) bin_off[i] = hk * kLocalGroups + 4 * gh + ((i + tau) & 3);

  const int n_tiles = (t_end - t_begin + kTile - 1) / kTile;
  // With one CTA per SM (R = 2) nothing hides this CTA's tail, so the value codebook copy
  // starts as soon as the last key gather is done; with two per SM the other CTA covers it
  // and the early copy only costs registers (measured: Zipf batch 254 -> 248 us, 32K R = 2
  // 81.8 -> 80.9 us, 128K R = 1 +0.5-1 us).
  constexpr bool kEarlyValueCopy = C::kMinBlocks == 1;

  // Software pipeline over tiles.  Iteration t: key side of tile t -> cluster barrier (the
  // peer's partial scores of tile t have arrived; every warp's tile t-1 maximum is in
  // mslot) -> full scores and the warp's maxima of tile t into mslot -> raise the reference
  // max from tile t-1's maximum if needed -> weights and bin atomics of tile t-1 (scores and
  // value codes kept in registers for one iteration).  The only barrier of a tile is the
  // cluster barrier (each warp waits only for its own code copies); no CTA-wide max
  // reduction.
  float sp[C::kSteps];           // scores of the previous tile's tokens (head hk; -inf = none)
  uint32_t vw[C::kSteps][R];     // value code bytes of those tokens (groups 4 gh .. 4 gh + 3)
#pragma unroll
  for (int st = 0; st < C::kSteps; ++st) {
    sp[st] = -INFINITY;
#pragma unroll
    for (int r = 0; r < R; ++r) vw[st][r] = 0u;
  }

  auto bin_atomics = [&]() {
#pragma unroll
    for (int st = 0; st < C::kSteps; ++st) {
      float e;
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(sp[st] - m_ref));   // -inf -> 0
      l_acc += (gh == 0) ? e : 0.f;     // lanes k and k ^ 4 hold the same head
      // R = 1 skips the per-token branch: a token past the split end has weight 0 (score
      // -inf), so its atomics add 0 to some bin (measured: faster at R = 1, slower at R = 2)
      if (R == 1 || sp[st] != -INFINITY) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t rot = __funnelshift_r(vw[st][r], vw[st][r], 8 * tau);  // byte i: group 4gh + ((i + tau) & 3)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = static_cast<int>(__byte_perm(rot, 0u, 0x4440u + i));
            const int bi = r * (kCodes * kHeads * kLocalGroups) + c * (kHeads * kLocalGroups) + bin_off[i];
            if (in_bounds(a.fault, bi, C::kBins)) atomicAdd(bins + bi, e);
          }
        }
      }
    }
  };

  // Raise the reference max of head hk to the maximum mt of a finished tile when mt exceeds
  // it by more than the slack, rescaling bins and l.  Every warp reads the same mt values
  // (lanes cover all 4 heads), so the branch is uniform over the CTA, and both CTAs of the
  // pair hold bit-identical scores, so they decide alike.  The caller guarantees that every
  // atomic already issued has completed (a CTA-wide barrier since) and that none of the
  // tile's own atomics has started.
  auto raise_ref = [&](float mt) {
    const bool raise = (m_ref == -INFINITY && mt != -INFINITY) || (mt > m_ref + kRescaleSlack);
    if (__any_sync(0xffffffffu, raise)) {
      const float m_new = raise ? mt : m_ref;
      const float f = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - m_new);
      // bins hold nothing before the first raise of every head: rescale only once some
      // head had a finite reference
      const bool rescale = __any_sync(0xffffffffu, m_ref != -INFINITY);
      l_acc *= f;
      m_ref = m_new;
      if (rescale) {
        if (tid < kHeads) fh[tid] = f;       // thread tid < 4 is lane tid: head tid
        __syncthreads();
        for (int i = tid; i < C::kBins; i += C::kThreads) bins[i] *= fh[(i >> 3) & 3];
        __syncthreads();
      }
    }
  };

  // one tile: FULL = every token of the tile is inside the split (no per-token checks)
  auto run_tile = [&](const int t_tile, const int tile, const int buf, auto full_tag, const bool last) {
    constexpr bool FULL = decltype(full_tag)::value;
    const uint8_t* cb = code_s + static_cast<size_t>(buf) * kTile * R * 16;
    float* xb = xchg + buf * (kTile * kHeads);
    float* pxb = peer_xchg + buf * (kTile * kHeads);

#pragma unroll
    for (int p = 0; p < 4; ++p) ph[p] = phase_at(f_s[4 * k + (p ^ (2 * fk))], t_tile + sigma);
    float s_part[C::kSteps];
    constexpr int kGS = C::kSteps >= 4 ? 4 : C::kSteps;   // steps per pass group
#pragma unroll
    for (int sg = 0; sg < C::kSteps; sg += kGS) {
      float pv[kGS][kHeads];
#pragma unroll
      for (int u = 0; u < kGS; ++u) {
        const int tt = (sg + u) * C::kSlots + sigma;
        float2 kw[4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int c = cb[(tt * R + r) * 16 + k];
          const int ci = ((r * kCodes + c) * kLocalGroups + k) * 2;
          const float4* src = cw_s + (in_bounds(a.fault, ci + 1, C::kCodeChunks) ? ci : 0);
          const float4 lo = src[fk], hi = src[fk ^ 1];
          if (r == 0) {
            kw[0] = make_float2(lo.x, lo.y); kw[1] = make_float2(lo.z, lo.w);
            kw[2] = make_float2(hi.x, hi.y); kw[3] = make_float2(hi.z, hi.w);
          } else {
            kw[0] = __fadd2_rn(kw[0], make_float2(lo.x, lo.y));
            kw[1] = __fadd2_rn(kw[1], make_float2(lo.z, lo.w));
            kw[2] = __fadd2_rn(kw[2], make_float2(hi.x, hi.y));
            kw[3] = __fadd2_rn(kw[3], make_float2(hi.z, hi.w));
          }
        }
        float2 part2[kHeads];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 x = cmul(ph[p], kw[p]);
#pragma unroll
          for (int j = 0; j < kHeads; ++j)
            part2[j] = p == 0 ? __fmul2_rn(qv[j][p], x) : __ffma2_rn(qv[j][p], x, part2[j]);
          ph[p] = cmul(ph[p], adv[p]);
        }
#pragma unroll
        for (int j = 0; j < kHeads; ++j) pv[u][j] = part2[j].x + part2[j].y;
      }
#pragma unroll
      for (int u = 0; u < kGS; ++u) {
        const int tt = (sg + u) * C::kSlots + sigma;
        const float r0 = pv[u][0] + __shfl_xor_sync(0xffffffffu, pv[u][2], 2);
        const float r1 = pv[u][1] + __shfl_xor_sync(0xffffffffu, pv[u][3], 2);
        float v = r0 + __shfl_xor_sync(0xffffffffu, r1, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        s_part[sg + u] = v;
        if (k < 4 && in_bounds(a.fault, tt * kHeads + hk, kTile * kHeads)) pxb[tt * kHeads + hk] = v;
      }
    }
    cluster_arrive_release();
    cluster_wait_acquire();             // the peer's partials of this tile are in xb
    if (kEarlyValueCopy && last && warp == 0) {
      // every thread of the CTA is past its last key gather: bring in the value codewords
      // over the key codewords now, behind this tile's softmax, bins and the l reduction
      // (the fence orders the gathers before the TMA writes)
      fence_proxy_async_smem();
      stage_codebook_tma<R>(cw_s, &a.val_map, rank, a.val_cb_stride == 0 ? 0 : h, tma_bar);
    }

    // full scores (the same order of addition in both CTAs -> identical values)
    float sc[C::kSteps];
    uint32_t vn[C::kSteps][R];
    float mx = -INFINITY;
#pragma unroll
    for (int st = 0; st < C::kSteps; ++st) {
      const int tt = st * C::kSlots + sigma;
      const float other = xb[tt * kHeads + hk];
      const float v = rank == 0 ? s_part[st] + other : other + s_part[st];
      sc[st] = (FULL || t_tile + tt < t_end) ? v : -INFINITY;
      mx = fmaxf(mx, sc[st]);
#pragma unroll
      for (int r = 0; r < R; ++r)
        vn[st][r] = *reinterpret_cast<const uint32_t*>(cb + (tt * R + r) * 16 + 8 + 4 * gh);
    }
    // this warp's maximum per head into the tile's slot (lanes 0..3: heads 0..3); the
    // slot two tiles back, read by every warp before this tile's cluster barrier, is reset
    // for the next tile
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (lane < kHeads) atomicMax(mslot + (tile % 3) * kHeads + lane, ord_of(mx));
    if (tid < kHeads) mslot[((tile + 1) % 3) * kHeads + tid] = ord_of(-INFINITY);
    if (tile > 0) {
      // every warp's maximum of the previous tile landed before this tile's cluster
      // barrier, and so did every atomic issued before it
      raise_ref(float_of_ord(mslot[((tile + 2) % 3) * kHeads + hk]));
      bin_atomics();                    // previous tile
    }
#pragma unroll
    for (int st = 0; st < C::kSteps; ++st) {
      sp[st] = sc[st];
#pragma unroll
      for (int r = 0; r < R; ++r) vw[st][r] = vn[st][r];
    }
  };

  for (int tile = 0; tile < n_tiles; ++tile) {
    const int t_tile = t_begin + tile * kTile;
    const int buf = tile & 1;
    if (tile > 0) {
      cp_async_wait_all();      // this warp's codes of this tile (issued one tile ago) landed
      __syncwarp();             // ... for every lane; the warp is done with the other buffer
    }
    if (tile + 1 < n_tiles) stage_codes(t_tile + kTile, buf ^ 1);
    if (t_tile + kTile <= t_end) {
      run_tile(t_tile, tile, buf, std::integral_constant<bool, true>(), tile + 1 == n_tiles);
    } else {
      run_tile(t_tile, tile, buf, std::integral_constant<bool, false>(), tile + 1 == n_tiles);
    }
  }
  // the last tile: its maxima are complete once every warp is past its scores
  __syncthreads();
  raise_ref(float_of_ord(mslot[((n_tiles - 1) % 3) * kHeads + hk]));
  bin_atomics();

  // ---- l: lanes hold disjoint shares of head hk; sum over slots, halves and warps ----
  l_acc += __shfl_xor_sync(0xffffffffu, l_acc, 4);
  l_acc += __shfl_xor_sync(0xffffffffu, l_acc, 8);
  l_acc += __shfl_xor_sync(0xffffffffu, l_acc, 16);
  __syncthreads();                                   // every bin update is done
  if (lane < kHeads) red[warp * kHeads + lane] = l_acc;
  __syncthreads();
  if (rank == 0 && tid < kHeads && parts_ok) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) v += red[w * kHeads + tid];
    a.part_l[part_row + static_cast<size_t>(tid) * a.n_splits] = v;
    a.part_m[part_row + static_cast<size_t>(tid) * a.n_splits] = m_ref * kLn2;   // lane tid: head tid
  }

  // ---- epilogue: o[head][8 G + d] = sum_{r,c} bins[r][c][head][G] * val_cb[G][r][c][d] ----
  // the value codewords of this CTA's groups, over the key codewords in the same layout
  // (copied since the last tile's cluster barrier if kEarlyValueCopy; else now: every read
  // of the key codewords happened before the barrier above, the fence orders them before
  // the TMA writes)
  if (!kEarlyValueCopy && warp == 0) {
    fence_proxy_async_smem();
    stage_codebook_tma<R>(cw_s, &a.val_map, rank, a.val_cb_stride == 0 ? 0 : h, tma_bar);
  }
  if (!mbar_wait(tma_bar, 1) && tid == 0) atomicOr(a.fault, kFaultCopyTimeout);
  {
    // warp = slice of codes, lane = (head, local group): bins reads are 32 consecutive
    // floats; codeword reads take chunk fv first (dims 4 fv .. 4 fv + 3 in acc[0..3]) so
    // that the 8 groups hit 8 distinct bank quads
    const int gl = lane & 7, hh = lane >> 3, fv = gl >> 2;
    constexpr int kPerSlice = R * kCodes / C::kWarps;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int ci = 0; ci < kPerSlice; ++ci) {
      const int rc = warp * kPerSlice + ci;            // r * 256 + c
      const float wgt = bins[(rc * kHeads + hh) * kLocalGroups + gl];
      const float4 v0 = cw_s[(rc * kLocalGroups + gl) * 2 + fv];
      const float4 v1 = cw_s[(rc * kLocalGroups + gl) * 2 + (fv ^ 1)];
      acc[0] = fmaf(wgt, v0.x, acc[0]); acc[1] = fmaf(wgt, v0.y, acc[1]);
      acc[2] = fmaf(wgt, v0.z, acc[2]); acc[3] = fmaf(wgt, v0.w, acc[3]);
      acc[4] = fmaf(wgt, v1.x, acc[4]); acc[5] = fmaf(wgt, v1.y, acc[5]);
      acc[6] = fmaf(wgt, v1.z, acc[6]); acc[7] = fmaf(wgt, v1.w, acc[7]);
    }
    __syncthreads();                                   // bins no longer read: reuse them
    float* part_s = bins;                              // [kWarps][32 lanes][8]
#pragma unroll
    for (int d = 0; d < 8; ++d) part_s[(warp * 32 + lane) * 8 + d] = acc[d ^ (4 * fv)];
    __syncthreads();
    for (int o = tid; o < kHeads * kLocalGroups * 8 && parts_ok; o += C::kThreads) {
      const int d = o & 7, ln = o >> 3;                // ln = head * 8 + local group
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < C::kWarps; ++w) v += part_s[(w * 32 + ln) * 8 + d];
      const int hh2 = ln >> 3, gl2 = ln & 7;
      a.part_o[(part_row + static_cast<size_t>(hh2) * a.n_splits) * kHeadDim +
               8 * (rank * kLocalGroups + gl2) + d] = v;
    }
  }
  // No cluster barrier is needed before leaving: the only distributed-shared-memory access
  // (the peer's partial-score stores into xchg) precedes the last tile's cluster barrier,
  // which both CTAs of the pair passed.
  if (a.counters != nullptr) merge_tail(a, b, h, hq0, kHeads, 2 * a.n_splits);
}

template <int R>
cudaError_t launch_gqa4(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = Cfg<R>::kSmem;
  auto k = decode_gqa4_kernel<R>;
  static PerDeviceFlag smem_set;
  cudaError_t e = set_smem_limit_once(smem_set, k, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(2 * a.n_splits, s.n_kv_heads, s.batch);
  k<<<grid, Cfg<R>::kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gqa4(const cvq_shape& s, const DecodeArgs& a, cudaStream_t stream) {
  return s.R == 1 ? launch_gqa4<1>(s, a, stream) : launch_gqa4<2>(s, a, stream);
}

}  // namespace cvq
