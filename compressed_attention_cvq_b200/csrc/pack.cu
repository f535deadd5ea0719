// cvq_pack_codes6: the paper's 6-bit codes (64-entry codebooks; CommVQ summary page, "Key
// results") from one byte per code to 4 codes in 3 bytes along every planar code row:
// codes 4i .. 4i+3 form the little-endian 24-bit word of bytes 3i .. 3i+2, code 4i + j in
// bits 6j .. 6j+5.  One thread per 4 codes: a 4-byte load, a 3-byte store.
#include "common.cuh"

namespace cvq {

namespace {

__global__ void pack_codes6_kernel(const uint8_t* __restrict__ in, uint8_t* __restrict__ out,
                                   size_t n_quads) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_quads;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    // rows are t_cap bytes (a multiple of 64) in and 3 t_cap / 4 out: quad i of the whole
    // tensor is 4 bytes in at 4 i and 3 bytes out at 3 i, whatever its row
    const uint32_t v = *reinterpret_cast<const uint32_t*>(in + 4 * i);
    const uint32_t w = (v & 63u) | (((v >> 8) & 63u) << 6) | (((v >> 16) & 63u) << 12) |
                       (((v >> 24) & 63u) << 18);
    uint8_t* o = out + 3 * i;
    o[0] = static_cast<uint8_t>(w);
    o[1] = static_cast<uint8_t>(w >> 8);
    o[2] = static_cast<uint8_t>(w >> 16);
  }
}

}  // namespace

cudaError_t launch_pack_codes6(const uint8_t* codes_in, uint8_t* packed_out, size_t rows, int t_cap,
                               cudaStream_t stream) {
  const size_t n_quads = rows * static_cast<size_t>(t_cap / 4);
  if (n_quads == 0) return cudaSuccess;
  const int threads = 256;
  const size_t want = (n_quads + threads - 1) / threads;
  const unsigned blocks = static_cast<unsigned>(want < 148u * 64u ? want : 148u * 64u);
  pack_codes6_kernel<<<blocks, threads, 0, stream>>>(codes_in, packed_out, n_quads);
  return cudaGetLastError();
}

}  // namespace cvq
