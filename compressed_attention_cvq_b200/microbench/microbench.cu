// Unit-throughput probes for the decode kernel's design on sm_100a: FP32 FMA (scalar
// and packed f32x2), the special-function unit (sin/cos, exp2), shared-memory 16-byte
// gathers with and without bank conflicts, shared-memory float atomics with distinct
// and random addresses, and warp shuffles.  Every access stays inside a fixed
// shared-memory array; every loop has a fixed trip count.
//
// C entry: cvqmb_run(kind, blocks, threads, iters, out, stream) launches one probe;
// the caller times it and divides the operation count by the time.
#include <cuda_runtime.h>
#include <stdint.h>

#define MB_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kChains = 8;

__global__ void ffma_kernel(float* out, int iters, float a, float b) {
  float x[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 1e-3f + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) x[i] = fmaf(x[i], a, b);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += x[i];
  if (s == 123.456f) out[threadIdx.x] = s;
}

__device__ __forceinline__ unsigned long long fma2(unsigned long long x, unsigned long long a,
                                                   unsigned long long b) {
  unsigned long long d;
  asm volatile("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(x), "l"(a), "l"(b));
  return d;
}

__global__ void ffma2_kernel(float* out, int iters, float a, float b) {
  unsigned long long x[kChains];
  float2 av = make_float2(a, a), bv = make_float2(b, b);
  const unsigned long long A = *reinterpret_cast<unsigned long long*>(&av);
  const unsigned long long B = *reinterpret_cast<unsigned long long*>(&bv);
#pragma unroll
  for (int i = 0; i < kChains; ++i) {
    float2 v = make_float2(threadIdx.x * 1e-3f + i, i * 0.5f);
    x[i] = *reinterpret_cast<unsigned long long*>(&v);
  }
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) x[i] = fma2(x[i], A, B);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) {
    float2 v = *reinterpret_cast<float2*>(&x[i]);
    s += v.x + v.y;
  }
  if (s == 123.456f) out[threadIdx.x] = s;
}

__global__ void sincos_kernel(float* out, int iters) {
  float x[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 1e-3f + i * 0.1f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) {
        float s, c;
        __sincosf(x[i], &s, &c);
        x[i] = s + c;
      }
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += x[i];
  if (s == 123.456f) out[threadIdx.x] = s;
}

__global__ void exp2_kernel(float* out, int iters) {
  float x[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) x[i] = -(threadIdx.x * 1e-3f + i * 0.1f);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) x[i] = exp2f(x[i]) - 1.0f;
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += x[i];
  if (s == 123.456f) out[threadIdx.x] = s;
}

// 16-byte gathers from a 32 KB shared array.  mode 0: a warp reads 32 consecutive
// 16-byte slots (conflict-free, 4 wavefronts); mode 1: pseudo-random 16-byte slots.
__global__ void lds128_kernel(float* out, int iters, int mode) {
  __shared__ float4 buf[2048];
  for (int i = threadIdx.x; i < 2048; i += blockDim.x) buf[i] = make_float4(i, i + 1, i + 2, i + 3);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  uint32_t rng = 2654435761u * (threadIdx.x + 1) + blockIdx.x * 97u;
  float4 acc = make_float4(0, 0, 0, 0);
  int idx = lane;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (mode == 0) {
        idx = ((idx + 41 * 32) & 2047 & ~31) | lane;
      } else {
        rng = rng * 1664525u + 1013904223u;
        idx = rng >> 21;
      }
      const float4 v = buf[idx];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
  }
  if (acc.x + acc.y + acc.z + acc.w == 123.456f) out[threadIdx.x] = acc.x;
}

// Shared float atomics (no return).  mode 0: each lane its own bank, mode 1: random
// addresses in a 4096-float region, mode 2: all lanes of a warp one address.
__global__ void red_kernel(float* out, int iters, int mode) {
  __shared__ float bins[4096];
  for (int i = threadIdx.x; i < 4096; i += blockDim.x) bins[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  uint32_t rng = 2654435761u * (threadIdx.x + 1) + blockIdx.x * 97u;
  int idx = lane;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (mode == 0) {
        idx = ((idx + 32 * 5) & 4095 & ~31) | lane;
      } else if (mode == 1) {
        rng = rng * 1664525u + 1013904223u;
        idx = rng >> 20;
      } else {
        idx = (threadIdx.x >> 5) * 32;
      }
      atomicAdd(&bins[idx], 1.0f);
    }
  }
  __syncthreads();
  if (bins[threadIdx.x] == 123.456f) out[threadIdx.x] = 1.f;
}

__global__ void shfl_kernel(float* out, int iters) {
  float x[4] = {threadIdx.x * 1.f, 1.f, 2.f, 3.f};
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] += __shfl_xor_sync(0xffffffffu, x[i], 1 << (r & 3));
    }
  }
  if (x[0] + x[1] + x[2] + x[3] == 123.456f) out[threadIdx.x] = x[0];
}

// Explicit shared reductions and plain read-modify-write, each lane on its own bank
// (mode 0: f32, 1: u32, 2: u64 (8-byte aligned, lanes on distinct 8-byte slots),
//  3: plain ld/add/st f32, 4: plain float4 ld/add/st conflict-free, 5: float4 gather
//  + two f32 reductions per iteration (mixed), 6: red.shared::cluster.add.f32 on this CTA's
//  own shared memory (the distributed-shared-memory form of the reduction))
__global__ void rmw_kernel(float* out, int iters, int mode) {
  __shared__ float4 buf[2048];
  float* bf = reinterpret_cast<float*>(buf);
  for (int i = threadIdx.x; i < 8192; i += blockDim.x) bf[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int idx = lane;
  float4 acc = make_float4(0, 0, 0, 0);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      idx = ((idx + 32 * 7) & 2047 & ~31) | lane;
      if (mode == 0) {
        unsigned a = (unsigned)__cvta_generic_to_shared(bf + idx);
        asm volatile("red.shared.add.f32 [%0], %1;" :: "r"(a), "f"(1.0f) : "memory");
      } else if (mode == 1) {
        unsigned a = (unsigned)__cvta_generic_to_shared(bf + idx);
        asm volatile("red.shared.add.u32 [%0], %1;" :: "r"(a), "r"(1u) : "memory");
      } else if (mode == 2) {
        unsigned a = (unsigned)__cvta_generic_to_shared(bf + 2 * idx);
        asm volatile("red.shared.add.u64 [%0], %1;" :: "r"(a), "l"(1ull) : "memory");
      } else if (mode == 3) {
        // each warp owns a private 32-float slice per round, so no two threads race
        float* p = bf + ((warp * 8 + r) & 255) * 32 + lane;
        *p += 1.0f;
      } else if (mode == 6) {
        unsigned a = (unsigned)__cvta_generic_to_shared(bf + idx);
        asm volatile("red.shared::cluster.add.f32 [%0], %1;" :: "r"(a), "f"(1.0f) : "memory");
      } else if (mode == 4) {
        float4* p = buf + (((warp * 8 + r) & 63) * 32 + lane);
        float4 v = *p;
        v.x += 1.f; v.y += 1.f; v.z += 1.f; v.w += 1.f;
        *p = v;
      } else {
        const float4 v = buf[idx];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        unsigned a = (unsigned)__cvta_generic_to_shared(bf + ((idx * 4 + 64) & 4095));  // + 1024 below stays < 8192
        asm volatile("red.shared.add.f32 [%0], %1;" :: "r"(a), "f"(1.0f) : "memory");
        asm volatile("red.shared.add.f32 [%0], %1;" :: "r"(a + 4096u), "f"(1.0f) : "memory");
      }
    }
  }
  __syncthreads();
  if (bf[threadIdx.x] + acc.x == 123.456f) out[threadIdx.x] = 1.f;
}

// Reductions into global memory (L2), each CTA in its own 64 KB window of `buf`
// (blocks x 16384 floats): mode 0: red.global.add.v4.f32 (16 bytes, one op) at
// pseudo-random 16-byte slots; 1: red.global.add.f32 at pseudo-random floats; 2: like 0,
// but every 5th op of a lane goes to one of 4 hot slots (a skewed code distribution).
__global__ void gred_kernel(float* buf, int iters, int mode) {
  float* win = buf + static_cast<size_t>(blockIdx.x) * 16384;
  unsigned x = 2654435761u * (threadIdx.x + 1) + 97u * blockIdx.x;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      x = x * 1664525u + 1013904223u;
      if (mode == 1) {
        float* p = win + (x >> 18);                         // 0 .. 16383
        asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(1.0f) : "memory");
      } else {
        unsigned slot = x >> 20;                            // 0 .. 4095
        if (mode == 2 && (r == 0 || r == 5)) slot &= 3u;    // 2 of 8 ops (25%) on 4 hot slots
        float* p = win + 4 * slot;
        asm volatile("red.global.add.v4.f32 [%0], {%1, %1, %1, %1};" ::"l"(p), "f"(1.0f) : "memory");
      }
    }
  }
}

// Value bins owned by one warp, updated without atomics (one 16-byte read-add-write adds a
// token's weights of 4 heads to the bin of its code): each warp owns 64 float4 bins, each
// lane takes one (token, group) per operation -- its code byte and its 4 weights from
// shared memory -- and lanes holding the same code take turns (__match_any_sync, rank
// among equal codes, one pass per rank, __syncwarp between passes).  skew = 0: codes
// uniform over 64; skew = 1: a quarter of them 0 (a hot code).  One op = one (token, group)
// update of 4 heads.  Indexes: bins (warp & 31) * 64 + code < 2048, weights < 256, codes
// < 8192.
__global__ void owned_bins_kernel(float* out, int iters, int skew) {
  __shared__ float4 bins[2048];
  __shared__ float4 wts[256];
  __shared__ uint8_t codes[8192];
  unsigned x = 2654435761u * (threadIdx.x + 1) + 97u * blockIdx.x;
  for (int i = threadIdx.x; i < 2048; i += blockDim.x) bins[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = threadIdx.x; i < 256; i += blockDim.x) wts[i] = make_float4(1.f, 0.5f, 0.25f, 0.125f);
  for (int i = threadIdx.x; i < 8192; i += blockDim.x) {
    x = x * 1664525u + 1013904223u;
    int c = static_cast<int>(x >> 26);
    if (skew && ((x >> 20) & 3u) == 0u) c = 0;
    codes[i] = static_cast<uint8_t>(c);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  float4* mine = bins + ((threadIdx.x >> 5) & 31) * 64;
  const unsigned below = (1u << lane) - 1u;
  int pos = (threadIdx.x >> 5) * 32 + lane;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      pos = (pos + 32 * 9) & 8191;
      const int c = codes[pos] & 63;
      const float4 w = wts[pos & 255];
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(peers & below);
      const int passes = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(rank));
      for (int k = 0; k <= passes; ++k) {
        if (rank == k) {
          float4 v = mine[c];
          v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
          mine[c] = v;
        }
        __syncwarp();
      }
    }
  }
  __syncthreads();
  if (bins[threadIdx.x & 2047].x == 123.456f) out[threadIdx.x] = 1.f;
}

}  // namespace

// kind: 0 ffma, 1 ffma2, 2 sincos, 3 exp2, 4 lds128 conflict-free, 5 lds128 random,
//       6 atomic distinct banks, 7 atomic random, 8 atomic same address, 9 shfl,
//       10..15 rmw_kernel modes 0..5 (mode 5 counts one gather + two reductions as one op),
//       16..18 gred_kernel modes 0..2 (`out` must hold blocks x 16384 floats),
//       19 rmw_kernel mode 6, 20..21 owned_bins_kernel skew 0..1 (blockDim <= 1024)
// Returns the operation count of the launch (per-thread ops x threads x blocks), or
// -1 for an unknown kind / launch error.  Operations: FMA lanes (ffma2 counts 2 per
// instruction), sin+cos pairs, exp2, 16-byte loads, atomics, shuffles.
MB_API double cvqmb_run(int kind, int blocks, int threads, int iters, float* out, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const double nt = static_cast<double>(blocks) * threads;
  double per = 0;
  switch (kind) {
    case 0: ffma_kernel<<<blocks, threads, 0, s>>>(out, iters, 0.999f, 1e-3f); per = 16.0 * kChains * iters; break;
    case 1: ffma2_kernel<<<blocks, threads, 0, s>>>(out, iters, 0.999f, 1e-3f); per = 32.0 * kChains * iters; break;
    case 2: sincos_kernel<<<blocks, threads, 0, s>>>(out, iters); per = 8.0 * kChains * iters; break;
    case 3: exp2_kernel<<<blocks, threads, 0, s>>>(out, iters); per = 16.0 * kChains * iters; break;
    case 4: lds128_kernel<<<blocks, threads, 0, s>>>(out, iters, 0); per = 8.0 * iters; break;
    case 5: lds128_kernel<<<blocks, threads, 0, s>>>(out, iters, 1); per = 8.0 * iters; break;
    case 6: red_kernel<<<blocks, threads, 0, s>>>(out, iters, 0); per = 8.0 * iters; break;
    case 7: red_kernel<<<blocks, threads, 0, s>>>(out, iters, 1); per = 8.0 * iters; break;
    case 8: red_kernel<<<blocks, threads, 0, s>>>(out, iters, 2); per = 8.0 * iters; break;
    case 9: shfl_kernel<<<blocks, threads, 0, s>>>(out, iters); per = 32.0 * iters; break;
    case 10: case 11: case 12: case 13: case 14: case 15:
      rmw_kernel<<<blocks, threads, 0, s>>>(out, iters, kind - 10); per = 8.0 * iters; break;
    case 19:
      rmw_kernel<<<blocks, threads, 0, s>>>(out, iters, 6); per = 8.0 * iters; break;
    case 20: case 21:
      if (threads > 1024) return -1;
      owned_bins_kernel<<<blocks, threads, 0, s>>>(out, iters, kind - 20); per = 8.0 * iters; break;
    case 16: case 17: case 18:
      gred_kernel<<<blocks, threads, 0, s>>>(out, iters, kind - 16); per = 8.0 * iters; break;
    default: return -1;
  }
  if (cudaGetLastError() != cudaSuccess) return -1;
  return per * nt;
}
