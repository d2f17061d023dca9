// Definitions shared by the kernels of the quantized linear library.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace sq {

constexpr int SQ_MAX_SEG = 16;

// 1.5 * 2^23: adding it to a value of magnitude below 2^22 leaves, in the
// fp32 bit pattern's low bits, that value rounded half-to-even to an integer.
constexpr float kMagic = 12582912.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;

// 1.5 * 2^19, whose fp32 unit in the last place is 2^-4: an int32 accumulator
// seeded with these bits and fed weights scaled by 16 (int4 codes unpacked
// into the high nibble of each byte) holds the bits of 1.5 * 2^19 + acc, exact
// while |acc| < 2^18 (a 128-wide group of int8 x int4 products: |acc| <=
// 128 * 127 * 8).
constexpr float kMagicW4 = 786432.0f;
constexpr uint32_t kMagicW4Bits = 0x49400000u;

// Bits of the per-device status word.
constexpr unsigned int SQ_STATUS_TIMEOUT = 1u;
constexpr unsigned int SQ_STATUS_RANGE = 2u;

// The per-device status word (one copy per device that loads the library).
__device__ unsigned int g_status;

__device__ __forceinline__ void raise_status(unsigned int bits) { atomicOr(&g_status, bits); }

// K-segment bounds passed by value: count segments, count + 1 bounds.
struct SegBounds {
  int32_t count;
  int32_t b[SQ_MAX_SEG + 1];
  __host__ __device__ __forceinline__ int segment_of(int32_t k) const {
    int j = 0;
#pragma unroll 1
    for (int i = 1; i < count; ++i) j += (k >= b[i]) ? 1 : 0;
    return j;
  }
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

}  // namespace sq
