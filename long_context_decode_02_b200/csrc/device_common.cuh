// Device helpers shared by liblowram's kernels: element conversion, RoPE table lookup,
// block-wide reductions, scans and a radix select. Arithmetic of the method itself lives
// in the kernel files.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
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

// ------------------------------------------------------------------ evicted caches
// Original chunk index of stored chunk c of batch element b (c itself without eviction).
// An entry outside [0, P / C) is reported and replaced by 0, so no table is read out of
// bounds.
__device__ __forceinline__ int chunk_position(const Dims& dm, const int32_t* chunk_pos, int b,
                                              int c, int* status) {
  if (!chunk_pos) return c;
  const int v = chunk_pos[(size_t)b * dm.Nc + c];
  if (v < 0 || v >= dm.P / dm.C) {
    raise_status(status, kStatusDeviceCheck);
    return 0;
  }
  return v;
}
__device__ __forceinline__ int token_position(const Dims& dm, const int32_t* chunk_pos, int b,
                                              int t, int* status) {
  return chunk_pos ? chunk_position(dm, chunk_pos, b, t / dm.C, status) * dm.C + t % dm.C : t;
}

// Value of element j of an int4 residual row e of pair p: code * scale (exact in fp32).
__device__ __forceinline__ float int4_residual(const uint8_t* codes, const __half* scales,
                                               const Dims& dm, size_t row, int j) {
  const uint8_t byte = codes[row * (dm.d / 2) + (j >> 1)];
  const int q = (j & 1) ? (int)(byte >> 4) : (int)(byte & 15);
  return (float)(q >= 8 ? q - 16 : q) * __half2float(scales[row * (dm.d / kInt4Group) + j / kInt4Group]);
}

// ------------------------------------------------------------------ RoPE
// (cos, sin) of t * theta_i from the two-level tables by angle addition.
__device__ __forceinline__ float2 rope_cs32(const RopeTables& rt, int i, int t) {
  const float2 lo = rt.lo32[(t & (kRopeLo - 1)) * rt.half + i];
  const float2 hi = rt.hi32[(size_t)(t >> kRopeLoBits) * rt.half + i];
  return make_float2(fmaf(hi.x, lo.x, -hi.y * lo.y), fmaf(hi.y, lo.x, hi.x * lo.y));
}
// (cos, sin) combination of a hi and a lo table entry by angle addition.
__device__ __forceinline__ float2 rope_combine(float2 hi, float2 lo) {
  return make_float2(fmaf(hi.x, lo.x, -hi.y * lo.y), fmaf(hi.y, lo.x, hi.x * lo.y));
}
__device__ __forceinline__ double2 rope_cs64(const RopeTables& rt, int i, int t) {
  const double2 lo = rt.lo64[(t & (kRopeLo - 1)) * rt.half + i];
  const double2 hi = rt.hi64[(size_t)(t >> kRopeLoBits) * rt.half + i];
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

// ------------------------------------------------------------------ thread groups
// A group of whole warps, numbered from 0, synchronised either by __syncthreads (the
// whole block, id 0) or by named barrier `id` over `nt` threads. The helpers below must
// be called by every thread of the group.
struct Grp {
  int tid, nt, id;
  __device__ __forceinline__ void sync() const {
    if (id == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nt) : "memory");
  }
};
__device__ __forceinline__ Grp whole_block() { return Grp{(int)threadIdx.x, (int)blockDim.x, 0}; }

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

// Max over the group. `scratch`: 33 words of shared memory.
__device__ inline float group_max(const Grp& g, float v, float* scratch) {
  const int lane = g.tid & 31, wid = g.tid >> 5, nw = g.nt >> 5;
  v = warp_max(v);
  g.sync();
  if (lane == 0) scratch[wid] = v;
  g.sync();
  float r = lane < nw ? scratch[lane] : -INFINITY;
  return warp_max(r);
}

// Exclusive prefix sum of v over the group in thread order; *total gets the sum.
__device__ inline int group_exclusive_scan(const Grp& g, int v, int* scratch, int* total) {
  const int lane = g.tid & 31, wid = g.tid >> 5, nw = g.nt >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  g.sync();
  if (lane == 31) scratch[wid] = incl;
  g.sync();
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
  g.sync();
  const int res = scratch[wid] + incl - v;
  *total = scratch[32];
  g.sync();
  return res;
}

// Key of the k-th largest (1-based k, 1 <= k <= n) among n uint32 keys produced by
// key_of(i), by a most-significant-digit-first radix pass over 8-bit digits.
// `hist` holds 256 words and `bc` 4 words of shared memory.
template <typename KeyFn>
__device__ uint32_t group_kth_largest(const Grp& g, int n, int k, KeyFn key_of,
                                      unsigned* hist, unsigned* bc) {
  uint32_t prefix = 0, mask = 0;
  unsigned remaining = (unsigned)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = g.tid; i < 256; i += g.nt) hist[i] = 0;
    g.sync();
    for (int i = g.tid; i < n; i += g.nt) {
      const uint32_t key = key_of(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    g.sync();
    if (g.tid < 32) {
      // lane l owns digits 255-8l .. 248-8l (high digits first)
      const int lane = g.tid;
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
    g.sync();
    prefix |= bc[0] << shift;
    mask |= 255u << shift;
    remaining = bc[1];
    g.sync();
  }
  return prefix;
}

// Same as group_kth_largest, with warp-aggregated histogram updates: lanes of a warp
// holding the same digit add their count with one atomic. For key sets concentrated in
// few digits (scores sharing an exponent).
template <typename KeyFn>
__device__ uint32_t group_kth_largest_aggr(const Grp& g, int n, int k, KeyFn key_of,
                                           unsigned* hist, unsigned* bc) {
  uint32_t prefix = 0, mask = 0;
  unsigned remaining = (unsigned)k;
  const int lane = g.tid & 31;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = g.tid; i < 256; i += g.nt) hist[i] = 0;
    g.sync();
    for (int base = 0; base < n; base += g.nt) {
      const int i = base + g.tid;
      unsigned digit = 256u;
      if (i < n) {
        const uint32_t key = key_of(i);
        if ((key & mask) == prefix) digit = (key >> shift) & 255u;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (digit < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers));
    }
    g.sync();
    if (g.tid < 32) {
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
      if (before < remaining && incl >= remaining) {
        unsigned acc = before;
        for (int j = 0; j < 8; ++j) {
          const int dg = 255 - 8 * lane - j;
          const unsigned c = hist[dg];
          if (acc + c >= remaining) { bc[0] = (unsigned)dg; bc[1] = remaining - acc; break; }
          acc += c;
        }
      }
    }
    g.sync();
    prefix |= bc[0] << shift;
    mask |= 255u << shift;
    remaining = bc[1];
    g.sync();
  }
  return prefix;
}

// Sort n (a power of two) (key, idx) pairs in shared memory so that (key desc, idx asc)
// comes first.
__device__ inline void group_sort_desc(const Grp& g, float* key, int* idx, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = g.tid; t < n / 2; t += g.nt) {
        const int i = 2 * t - (t & (stride - 1));
        const int j = i + stride;
        const float ki = key[i], kj = key[j];
        const int ii = idx[i], ij = idx[j];
        const bool j_first = (kj > ki) || (kj == ki && ij < ii);
        const bool i_first = (ki > kj) || (ki == kj && ii < ij);
        const bool up = (i & size) == 0;
        if (up ? j_first : i_first) {
          key[i] = kj; key[j] = ki;
          idx[i] = ij; idx[j] = ii;
        }
      }
      g.sync();
    }
  }
}

// Ascending sort of n (power of two) ints in shared memory.
__device__ inline void group_sort_int_asc(const Grp& g, int* v, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = g.tid; t < n / 2; t += g.nt) {
        const int i = 2 * t - (t & (stride - 1));
        const int j = i + stride;
        const int a = v[i], b = v[j];
        const bool up = (i & size) == 0;
        if (up ? (b < a) : (a < b)) { v[i] = b; v[j] = a; }
      }
      g.sync();
    }
  }
}

}  // namespace lowram
