// cvq_attend_static: one decode step (the GQA decode with the fused split merge,
// cvq_attend) whose workspace -- split partial states and arrival counters -- is a fixed,
// file-scope device array instead of caller-allocated memory.
//
// For callers that cannot allocate device memory while decoding: a serving process whose
// memory pool has already claimed all free HBM for the KV cache, a plugin whose host
// hands it no allocator, or a decode loop that cannot pay for cudaMalloc's implicit
// synchronization.  They pass only inputs and outputs; the intermediate partial states
// go to g_static_scratch, which every GPU that loads this library holds until exit.
//
// Layout of the array (fixed, whatever the shape of a call):
//   [0, kCounterBytes)              arrival counters, one int32 per (sequence, query head);
//                                   no call ever writes partial states here
//   [kCounterBytes, kScratchBytes)  split partial states of the current call
// The counters a call uses are cleared on the call's stream before its decode kernel, so
// a call never depends on what an earlier call (of any shape) left in the array.
#include <mutex>

#include "common.cuh"

using namespace cvq;

namespace {

constexpr size_t kScratchBytes = CVQ_STATIC_SCRATCH_BYTES;
constexpr size_t kCounterBytes = CVQ_STATIC_COUNTER_BYTES;
constexpr size_t kCounterInts = kCounterBytes / sizeof(int);
static_assert(kScratchBytes % 256 == 0 && kCounterBytes % 256 == 0,
              "both regions keep 256-byte alignment");
static_assert(kCounterBytes < kScratchBytes, "the partial states need room after the counters");

// Counters, then the partial states of the most recent call.  In host code this name is
// only a stand-in for the symbol: its device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
unsigned char* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_static_scratch on the current device, looked up once per device
// (with that device current) and cached.
cudaError_t scratch_address(unsigned char** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" CVQ_API cvq_status cvq_attend_static(
    const cvq_shape* s, const void* q, int q_dtype, const float* key_cb,
    int64_t key_cb_head_stride, const uint8_t* key_codes, const uint8_t* val_codes,
    const int32_t* seq_lens, const float* val_cb, int64_t val_cb_head_stride, int n_splits,
    float* out, float* lse, void* stream) {
  if (out == nullptr || lse == nullptr) return CVQ_ERR_NULL;
  if (!aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return CVQ_ERR_ALIGN;
  if (s == nullptr) return CVQ_ERR_NULL;
  if (n_splits < 1 || n_splits > 4096) return CVQ_ERR_WORKSPACE;
  if (s->batch < 1 || s->n_q_heads < 1) return CVQ_ERR_SHAPE;
  const size_t parts = cvq_partials_bytes(s, n_splits);
  if (parts == 0)   // an invalid shape: cvq_attend reports which check fails, before any launch
    return cvq_attend(s, q, q_dtype, key_cb, key_cb_head_stride, key_codes, val_codes, seq_lens,
                      val_cb, val_cb_head_stride, n_splits, nullptr, out, lse, stream);
  const size_t n_counters = static_cast<size_t>(s->batch) * s->n_q_heads;
  if (parts > kScratchBytes - kCounterBytes || n_counters > kCounterInts) return CVQ_ERR_STATIC_LIMIT;

  unsigned char* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return CVQ_ERR_CUDA;
  int* counters = reinterpret_cast<int*>(base);
  float* partials = reinterpret_cast<float*>(base + kCounterBytes);
  // The arrival counters must start at zero.  A completed call leaves its counters zero,
  // but the call clears them anyway (an asynchronous memset on its stream, after every
  // argument check and before the decode kernel; it allocates nothing), so that it does not
  // depend on any earlier call: one of another shape, or one whose kernel never completed.
  return attend_into(s, q, q_dtype, key_cb, key_cb_head_stride, key_codes, val_codes, seq_lens,
                     val_cb, val_cb_head_stride, n_splits, partials, counters, out, lse, stream,
                     n_counters);
}
