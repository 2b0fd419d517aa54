// Weight preparation: MX FP4 scale bytes from row order into the scale-atom
// order the block-scaled tensor-core MMA reads (one 512-byte atom per 128 x
// 128 block: 32 TMEM lanes x 16 bytes, row r of the block in lane r % 32,
// word r / 32, byte b = its scale of block elements 32 b .. 32 b + 31).
#include "moe_internal.cuh"

namespace moe {
namespace {

// One thread per 16-byte lane row of an atom: the four words of rows
// r0, r0 + 32, r0 + 64, r0 + 96 (r0 = the atom's lane), one 4-byte load each
// (the four group scales of one row are consecutive in row order).
__global__ void pack_mx_scales_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                      int64_t atoms, int64_t rblocks, int64_t kblocks, int64_t groups) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // atom * 32 + lane
  if (i >= atoms * 32) return;
  const int64_t atom = i >> 5;
  const int lane = (int)(i & 31);
  const int64_t kb = atom % kblocks;
  const int64_t rb = (atom / kblocks) % rblocks;
  const int64_t mat = atom / (kblocks * rblocks);
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t row = (mat * rblocks + rb) * 128 + j * 32 + lane;
    const uint8_t* p = src + row * groups + kb * 4;   // groups % 4 == 0: 4-byte aligned
    w[j] = __ldg(reinterpret_cast<const uint32_t*>(p));
  }
  reinterpret_cast<uint4*>(dst + atom * kSfAtomBytes)[lane] = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_pack_mx_scales(int64_t n, int64_t rows, int64_t cols, const void* src, void* dst,
                                         moe_stream_t stream) {
  using namespace moe;
  if (n < 0 || rows < 0 || cols < 0 || rows % 128 != 0 || cols % 128 != 0) return MOE_ERR_INVALID_ARG;
  if (n == 0 || rows == 0 || cols == 0) return MOE_OK;
  if (!src || !dst || !aligned16(dst) || ((uintptr_t)src & 3u) != 0) return MOE_ERR_INVALID_ARG;
  if (rows > (int64_t)1 << 30 || cols > (int64_t)1 << 30 || n > (int64_t)1 << 20) return MOE_ERR_INVALID_ARG;
  const int64_t rblocks = rows / 128, kblocks = cols / 128;
  const int64_t atoms = n * rblocks * kblocks;
  if (atoms > ((int64_t)1 << 40)) return MOE_ERR_INVALID_ARG;
  const int threads = 256;
  const int64_t blocks = (atoms * 32 + threads - 1) / threads;
  if (blocks > INT32_MAX) return MOE_ERR_INVALID_ARG;
  pack_mx_scales_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
      (const uint8_t*)src, (uint8_t*)dst, atoms, rblocks, kblocks, cols / 32);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
