// AWQ int4 packing and unpacking (GPTQModel wiki page "ParoQuant", section
// "Stored tensors": qweight (I, O//8), qzeros (I//G, O//8), INT32 words of
// eight 4-bit codes).  Nibble order inside a word follows the public AWQ
// convention: nibble t (bits 4t..4t+3) of word w holds column 8w + ORDER[t],
// ORDER = {0,2,4,6,1,3,5,7} — so extracting (word >> 4j) & 0x000F000F yields
// the adjacent columns (2j, 2j+1) as the two halves of a 32-bit register.
#pragma once

#include "common.cuh"

namespace paro {

// nibble position of column c (inverse of ORDER)
__device__ __forceinline__ int awq_nibble_of_column(int c) { return (c >> 1) + 4 * (c & 1); }

// src: uint8 [N, R] (column n, row r) -> dst: int32 [R, N/8].
// grid (ceil(R/256), N/8), block 256; thread = one output word, r fastest so the
// byte reads of one column are coalesced across the warp.
__global__ void pack_rows_kernel(const uint8_t* __restrict__ src, int32_t* __restrict__ dst,
                                 int64_t N, int64_t R) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t w = blockIdx.y;
  if (r >= R) return;
  uint32_t word = 0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t code = src[(8 * w + c) * R + r] & 0xFu;
    word |= code << (4 * awq_nibble_of_column(c));
  }
  dst[r * (N / 8) + w] = static_cast<int32_t>(word);
}

// Inverse: dst int32 [R, N/8] -> src uint8 [N, R].
__global__ void unpack_rows_kernel(const int32_t* __restrict__ dst, uint8_t* __restrict__ src,
                                   int64_t N, int64_t R) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t w = blockIdx.y;
  if (r >= R) return;
  const uint32_t word = static_cast<uint32_t>(dst[r * (N / 8) + w]);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    src[(8 * w + c) * R + r] = static_cast<uint8_t>((word >> (4 * awq_nibble_of_column(c))) & 0xFu);
}

}  // namespace paro
