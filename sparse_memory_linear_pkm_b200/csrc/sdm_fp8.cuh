// Block-scaled fp8 state (sm_100a): E4M3 values with one power-of-two scale
// per 16 consecutive values of a state row. The pages ask for int8/fp8
// quantisation of the state at N = 10^7 (SDM explainer, "工程落地关键点", item
// 2) without fixing a format; this one is OCP FP8 E4M3 (bias 7, subnormals
// down to 2^-9, largest finite 448, no infinities, S.1111.111 never produced)
// scaled in blocks of 16 as the OCP MX formats do in blocks of 32: codes =
// round-to-nearest-even(x / 2^e), and for a block whose largest magnitude is
// m > 0, e is the smallest integer for which that rounding of m / 2^e stays at
// most 448, i.e. the smallest e with m <= 464 * 2^e (464, halfway between 448
// and the next step 480, rounds to the even 448), clamped to the int8 range;
// an all-zero block has e = 0. So no value is ever clamped, and re-quantising
// a decoded block gives back the same codes and exponent. Every scaling is by
// a power of two, exact in fp32, so the code decisions depend only on the
// fp32 values being quantised.
//
// Layout of a state of R rows of d_v values: R * d_v code bytes, then
// R * d_v / 16 exponent bytes (int8).
#pragma once

#include <cuda_fp8.h>

#include "sdm_device.cuh"

namespace sdm {

struct Fp8Blk {};  // state-type tag of the block-scaled fp8 state: one code byte per value
static_assert(sizeof(Fp8Blk) == 1, "Fp8Blk pointers step over code bytes");

// 2^e as an fp32 for e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2f(int e) {
  return e >= -126 ? __int_as_float((e + 127) << 23) : __int_as_float(1 << 22);
}

// Decodes one 16-byte unit of codes (value i in byte i) with its block
// exponent. The E4M3 -> half conversion is exact (every E4M3 value is a half).
__device__ __forceinline__ void fp8blk_unpack16(const uint4& u, int ex, float* out) {
  const float s = pow2f(ex);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_fp8x2_storage_t p = static_cast<__nv_fp8x2_storage_t>((w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(p, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
    out[2 * i] = f.x * s;
    out[2 * i + 1] = f.y * s;
  }
}

// Quantises 16 fp32 values into one unit of codes; returns the exponent. The
// division by 2^e is exact; the conversion rounds to nearest even and
// saturates to +-448 (the format's definition).
__device__ __forceinline__ int fp8blk_pack16(const float* x, uint4* u) {
  float mx = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(x[i]));
  int e = 0;
  if (mx > 0.0f) {
    int k;
    const float f = frexpf(mx, &k);            // mx = f * 2^k, f in [0.5, 1): mx / 2^(k-9) = 512 f
    e = (k - 9) + (f > 0.90625f ? 1 : 0);      // 512 f > 464: one binade up
    e = min(127, max(-127, e));
  }
  const float inv = pow2f(-e);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_fp8x2_storage_t p =
        __nv_cvt_float2_to_fp8x2(make_float2(x[2 * i] * inv, x[2 * i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
    w[i >> 1] |= static_cast<uint32_t>(p) << (16 * (i & 1));
  }
  *u = make_uint4(w[0], w[1], w[2], w[3]);
  return e;
}

// codes[16 b .. 16 b + 15], exps[b] <- the quantised block b of x.
static __global__ void __launch_bounds__(256) k_quantize_fp8blk(const float* __restrict__ x, int64_t n_blocks,
                                                         uint8_t* __restrict__ codes, int8_t* __restrict__ exps) {
  for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < n_blocks;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v[16];
    const float4* src = reinterpret_cast<const float4*>(x + b * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = src[i];
      v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    uint4 u;
    const int e = fp8blk_pack16(v, &u);
    reinterpret_cast<uint4*>(codes)[b] = u;
    exps[b] = static_cast<int8_t>(e);
  }
}

}  // namespace sdm
