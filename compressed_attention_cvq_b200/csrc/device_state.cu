// Host side of the TMA codebook staging and the library's device fault word.
//
// encode_codebook_map builds the tiled tensor map through which the 4-query-head decode
// kernel copies its half of a codebook into shared memory (8 TMA copies per round).  The
// map's dimensions, innermost first, are
//   d0: the 8 floats of a codeword    (contiguous, 32 B)
//   d1: group (16)                    stride R * 256 * 32 B
//   d2: round * 256 + code (R * 256)  stride 32 B
//   d3: head                          stride head_stride * 4 B
// and the box {8, 8, kCodeBoxRows, 1} lands in shared memory in the order
// [code][local group][8 floats]: one token's 8 groups are 8 consecutive 32-byte
// codewords, and the kernel's lanes 0-3 / 4-7 read their lower / upper 16-byte halves
// first, which puts the 8 loads of a token in 8 distinct bank quads.
//
// The fault word is a device variable that kernels OR bits into when a bounded wait gives
// up (a copy that never completed); cvq_fault_status reads it.
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"

using namespace cvq;

namespace {

__device__ unsigned int g_fault_word;

constexpr int kMaxDevices = 128;
unsigned int* g_fault_addr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_mu;

cudaError_t encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                           cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = g_encode;
  return cudaSuccess;
}

}  // namespace

namespace cvq {

// A map depends only on (base, head stride, heads, R): the last kMapCache maps encoded are
// kept, so a decode loop over the same codebooks does not re-encode them every call.
namespace {
constexpr int kMapCache = 16;
struct MapEntry {
  const float* base = nullptr;
  long long head_stride = 0;
  int n_heads = 0, R = 0;
  bool valid = false;
  CUtensorMap map;
};
MapEntry g_map_cache[kMapCache];
int g_map_next = 0;
}  // namespace

cudaError_t encode_codebook_map(CUtensorMap* map, const float* base, long long head_stride,
                                int n_heads, int R) {
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (const MapEntry& m : g_map_cache) {
      if (m.valid && m.base == base && m.head_stride == head_stride && m.n_heads == n_heads && m.R == R) {
        *map = m.map;
        return cudaSuccess;
      }
    }
  }
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  cudaError_t e = encoder(&enc);
  if (e != cudaSuccess) return e;
  const cuuint64_t per_head = static_cast<cuuint64_t>(kGroups) * R * kCodes * kCodeword;   // floats
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kCodeword), static_cast<cuuint64_t>(kGroups),
                              static_cast<cuuint64_t>(R) * kCodes,
                              head_stride == 0 ? 1u : static_cast<cuuint64_t>(n_heads)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(R) * kCodes * kCodeword * sizeof(float),
                                 kCodeword * sizeof(float),
                                 (head_stride == 0 ? per_head : static_cast<cuuint64_t>(head_stride)) *
                                     sizeof(float)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(kCodeword), 8, static_cast<cuuint32_t>(kCodeBoxRows), 1};
  const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(base), dims, strides,
                         box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lock(g_mu);
  MapEntry& slot = g_map_cache[g_map_next];
  g_map_next = (g_map_next + 1) % kMapCache;
  slot.base = base;
  slot.head_stride = head_stride;
  slot.n_heads = n_heads;
  slot.R = R;
  slot.map = *map;
  slot.valid = true;
  return cudaSuccess;
}

cudaError_t fault_word_address(unsigned int** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_fault_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fault_word);
    if (e != cudaSuccess) return e;
    g_fault_addr[dev] = static_cast<unsigned int*>(p);
  }
  *out = g_fault_addr[dev];
  return cudaSuccess;
}

}  // namespace cvq

extern "C" CVQ_API cvq_status cvq_fault_status(uint32_t* flags, int clear) {
  if (flags == nullptr) return CVQ_ERR_NULL;
  unsigned int* addr = nullptr;
  if (fault_word_address(&addr) != cudaSuccess) return CVQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, addr, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return CVQ_ERR_CUDA;
  if (clear && v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpy(addr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return CVQ_ERR_CUDA;
  }
  *flags = v;
  return CVQ_OK;
}
