// Device helpers shared by liblowram's kernels: element conversion, RoPE table lookup,
// block-wide reductions, scans and a radix select. Arithmetic of the method itself lives
// in the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "lowram_internal.h"

namespace lowram {

// ------------------------------------------------------------------ element access
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p, size_t i) { return to_f(p[i]); }

template <typename T>
__device__ __forceinline__ double ldd(const T* p, size_t i) { return (double)to_f(p[i]); }

// bf16 pair (low half first in memory) to two floats, exactly.
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Load E consecutive elements (E in {2, 4}; 8/16-byte aligned) as floats.
template <typename T, int E> struct VecLoad;
template <> struct VecLoad<__nv_bfloat16, 4> {
  __device__ static void load(const __nv_bfloat16* p, float* o) {
    uint2 w = *reinterpret_cast<const uint2*>(p);
    float2 a = bf2_to_f2(w.x), b = bf2_to_f2(w.y);
    o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
  }
};
template <> struct VecLoad<__nv_bfloat16, 2> {
  __device__ static void load(const __nv_bfloat16* p, float* o) {
    float2 a = bf2_to_f2(*reinterpret_cast<const uint32_t*>(p));
    o[0] = a.x; o[1] = a.y;
  }
};
template <> struct VecLoad<float, 4> {
  __device__ static void load(const float* p, float* o) {
    float4 a = *reinterpret_cast<const float4*>(p);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  }
};
template <> struct VecLoad<float, 2> {
  __device__ static void load(const float* p, float* o) {
    float2 a = *reinterpret_cast<const float2*>(p);
    o[0] = a.x; o[1] = a.y;
  }
};

// ------------------------------------------------------------------ status word
__device__ __forceinline__ void raise_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// ------------------------------------------------------------------ RoPE
// (cos, sin) of t * theta_i from the two-level tables by angle addition.
__device__ __forceinline__ float2 rope_cs32(const RopeTables& rt, int i, int t) {
  const float2 lo = rt.lo32[i * kRopeLo + (t & (kRopeLo - 1))];
  const float2 hi = rt.hi32[(size_t)i * rt.n_hi + (t >> kRopeLoBits)];
  return make_float2(fmaf(hi.x, lo.x, -hi.y * lo.y), fmaf(hi.y, lo.x, hi.x * lo.y));
}
__device__ __forceinline__ double2 rope_cs64(const RopeTables& rt, int i, int t) {
  const double2 lo = rt.lo64[i * kRopeLo + (t & (kRopeLo - 1))];
  const double2 hi = rt.hi64[(size_t)i * rt.n_hi + (t >> kRopeLoBits)];
  return make_double2(hi.x * lo.x - hi.y * lo.y, hi.y * lo.x + hi.x * lo.y);
}

// ------------------------------------------------------------------ activations
// Accurate forms (expf / erff), used by encode and the CUDA-core decode kernel.
__device__ __forceinline__ float act_f(float x, int act) {
  if (act == LOWRAM_ACT_SILU) return x / (1.0f + expf(-x));
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}
__device__ __forceinline__ double act_d(double x, int act) {
  if (act == LOWRAM_ACT_SILU) return x / (1.0 + exp(-x));
  return 0.5 * x * (1.0 + erf(x * 0.70710678118654752440));
}

// ------------------------------------------------------------------ ordering keys
// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t f2key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// ------------------------------------------------------------------ block reductions
// All helpers below must be called by every thread of the block; blockDim.x is a
// multiple of 32 and at most 1024. `scratch` is shared memory of at least 33 words.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ inline float block_max(float v, float* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) scratch[wid] = v;
  __syncthreads();
  float r = lane < nw ? scratch[lane] : -INFINITY;
  r = warp_max(r);
  return r;
}

// Exclusive prefix sum of v over the block in thread order; *total gets the sum.
__device__ inline int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __syncthreads();
  if (lane == 31) scratch[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int w = lane < nw ? scratch[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < nw) scratch[lane] = wi - w;  // exclusive warp offsets
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  const int res = scratch[wid] + incl - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}

// Key of the k-th largest (1-based k, 1 <= k <= n) among n uint32 keys produced by
// key_of(i), by a most-significant-digit-first radix pass over 8-bit digits.
// `hist` holds 256 words and `bc` 4 words of shared memory.
template <typename KeyFn>
__device__ uint32_t block_kth_largest(int n, int k, KeyFn key_of, unsigned* hist,
                                      unsigned* bc) {
  uint32_t prefix = 0, mask = 0;
  unsigned remaining = (unsigned)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t key = key_of(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255-8l .. 248-8l (high digits first)
      const int lane = threadIdx.x;
      unsigned own = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) own += hist[255 - 8 * lane - j];
      unsigned incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const unsigned before = incl - own;
      const bool here = before < remaining && incl >= remaining;
      if (here) {
        unsigned acc = before;
        for (int j = 0; j < 8; ++j) {
          const int dg = 255 - 8 * lane - j;
          const unsigned c = hist[dg];
          if (acc + c >= remaining) { bc[0] = (unsigned)dg; bc[1] = remaining - acc; break; }
          acc += c;
        }
      }
    }
    __syncthreads();
    prefix |= bc[0] << shift;
    mask |= 255u << shift;
    remaining = bc[1];
    __syncthreads();
  }
  return prefix;
}

}  // namespace lowram
