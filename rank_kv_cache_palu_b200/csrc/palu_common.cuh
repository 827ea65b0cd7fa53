// Shared device-side helpers of libpalu: dtype traits, the device status word,
// and the RoPE angle reduction.  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "palu.h"

namespace palu {

// ---------------------------------------------------------------- status word
// The first 256 bytes of every workspace.  Kernels record the first fault they
// see (bounds, timeout) here and skip the access instead of faulting.
struct DevStatus {
  int32_t code;    // palu_status value, 0 = OK
  int32_t detail;  // kernel-specific: which wait / which index
  int32_t pad[62];
};
static_assert(sizeof(DevStatus) == 256, "status header is 256 bytes");

__device__ __forceinline__ void report(DevStatus* st, int code, int detail) {
  if (st != nullptr && atomicCAS(&st->code, 0, code) == 0) st->detail = detail;
}

// ---------------------------------------------------------------- dtypes
template <int DT> struct Dt;
template <> struct Dt<PALU_F32> {
  using T = float;
  static constexpr int bytes = 4;
  __device__ __forceinline__ static float to_f(T v) { return v; }
  __device__ __forceinline__ static T from_f(float v) { return v; }
};
template <> struct Dt<PALU_F16> {
  using T = __half;
  static constexpr int bytes = 2;
  __device__ __forceinline__ static float to_f(T v) { return __half2float(v); }
  __device__ __forceinline__ static T from_f(float v) { return __float2half_rn(v); }
};
template <> struct Dt<PALU_BF16> {
  using T = __nv_bfloat16;
  static constexpr int bytes = 2;
  __device__ __forceinline__ static float to_f(T v) { return __bfloat162float(v); }
  __device__ __forceinline__ static T from_f(float v) { return __float2bfloat16_rn(v); }
};

// Entry of a column table (entry i owns columns [col[i], col[i + 1]), n entries)
// that holds column c; columns past the last entry map to the last one.
__host__ __device__ inline int col_entry(const uint16_t* col, int n, int c) {
  int e = 0;
  while (e + 1 < n && col[e + 1] <= c) ++e;
  return e;
}

// Bytes of one token's int4 scale row for rank r: r/32 fp16 scales, padded to 16.
__host__ __device__ inline long long int4_scale_row(int r) { return (2LL * (r / 32) + 15) / 16 * 16; }

// Decode latent entry j of token t from its (page, group) block `blk` of P
// tokens (swizzled layout; int4: code × fp16 scale from the token-major scale
// row `srow`, rounded to the compute dtype ACT exactly as the dequantised value
// the MMA path feeds).
__host__ __device__ inline long long swz_offset(int t, long long o, int P) {
  const long long b = o >> 7;
  const int unit = (int)((o >> 4) & 7) ^ (t & 7);
  return b * (long long)P * 128 + (long long)t * 128 + unit * 16 + (o & 15);
}

template <int LAT, int ACT>
__device__ __forceinline__ float load_latent(const uint8_t* blk, int t, int P, const uint8_t* srow, int j) {
  if constexpr (LAT == PALU_INT4) {
    const uint8_t byte = blk[swz_offset(t, j >> 1, P)];
    int code = (j & 1) ? (byte >> 4) : (byte & 0xF);
    code = (code ^ 8) - 8;  // sign-extend the 4-bit two's complement
    const float s = __half2float(reinterpret_cast<const __half*>(srow)[j >> 5]);
    return Dt<ACT>::to_f(Dt<ACT>::from_f(float(code) * s));
  } else {
    using T = typename Dt<LAT>::T;
    return Dt<LAT>::to_f(*reinterpret_cast<const T*>(blk + swz_offset(t, (long long)j * sizeof(T), P)));
  }
}

// ---------------------------------------------------------------- RoPE angles
// The angle of frequency i at integer position p is p·θ_i with θ_i =
// base^(-2i/d_h).  Its cosine and sine only need p·θ_i modulo 2π, i.e. the
// fractional part of p·ω_i with ω_i = θ_i/(2π).  The host passes ω_i as a
// 64-bit fixed-point fraction; the product with p modulo 2^64 is then exact
// integer arithmetic, and its top 32 bits give the turn in [-1/2, 1/2).
__device__ __forceinline__ float rope_turn(int32_t pos, uint64_t omega) {
  const uint32_t lo = static_cast<uint32_t>(omega);
  const uint32_t hi = static_cast<uint32_t>(omega >> 32);
  const uint32_t p = static_cast<uint32_t>(pos);
  uint32_t top = p * hi + __umulhi(p, lo);
  if (pos < 0) top -= lo;  // two's-complement extension of a negative position
  return static_cast<float>(static_cast<int32_t>(top)) * 0x1p-32f;
}

// Accurate cosine/sine of 2π·turn (CUDA-core path).
__device__ __forceinline__ void rope_cs_accurate(int32_t pos, uint64_t omega, float& c, float& s) {
  sincospif(2.0f * rope_turn(pos, omega), &s, &c);
}

// Fast cosine/sine of 2π·turn: the argument is already reduced to [-π, π), the
// range the hardware approximations are specified on (tensor-core path).
__device__ __forceinline__ void rope_cs_fast(int32_t pos, uint64_t omega, float& c, float& s) {
  const float a = rope_turn(pos, omega) * 6.28318530717958647692f;
  __sincosf(a, &s, &c);
}

}  // namespace palu
