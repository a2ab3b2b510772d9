// Kernel (b), CUDA-core form: reconstruct the selected chunks and attend over them,
// plus the split-K combine kernels used by both reconstruct-and-attend kernels.
//
// Method (LowRAM summary on agihunt.info, key paragraph and value-amortisation
// paragraph; cctest "How the method works": Low-rank keys, Amortised values,
// Residuals for difficult tokens, Selective reconstruction): for the selected chunks,
//   K~_pre,t = B_h c_t             (xKV basis rows of head h times the token's coefficients)
//   K~_rot,t = R(t) K~_pre,t       (RoPE re-applied at the token's position)
//   V~_t     = W2 act(W1 K~_pre,t + b1) + b2  (+ R_t when t holds a residual)
//   out_g    = softmax_t(q_g . K~_rot,t / sqrt d) V~_t   over the selected tokens only.
//
// This kernel is the fp32-accurate path (fp32 storage needs 1e-4 of output RMS, out of
// reach of bf16/tf32 tensor cores) and the general-shape path. One CTA reconstructs a
// tile of 32 tokens of one (batch, KV head) in shared memory, computes that tile's
// softmax statistics and weighted value sum for the G query heads, and writes them as a
// split-K partial; the combine kernel merges the tiles. Nothing rebuilt reaches HBM.
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace lowram {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtTT = 32;   // tokens per tile
constexpr int kMaxG = 8;

template <int D, int FH>
struct SimtSmem {
  static size_t floats(int r, int G) {
    return (size_t)kSimtTT * r + kSimtTT * D + kSimtTT * FH + kSimtTT * D + (size_t)G * D +
           (size_t)G * kSimtTT;
  }
};

template <typename T, int D, int FH>
__global__ void __launch_bounds__(kSimtThreads) attend_simt_kernel(const AttendArgs a) {
  const Dims& dm = a.dm;
  const int p = blockIdx.y, tile = blockIdx.x;
  const int b = p / dm.H, h = p % dm.H;
  const int r = dm.r, C = dm.C, G = dm.G, k = dm.k;
  const int tid = threadIdx.x;
  const int CPT = kSimtTT / C;

  extern __shared__ float sm[];
  float* cs = sm;                          // [TT][r]
  float* kp = cs + kSimtTT * r;            // [TT][D]   pre-RoPE rebuilt keys
  float* hid = kp + kSimtTT * D;           // [TT][FH]
  float* vv = hid + kSimtTT * FH;          // [TT][D]   reconstructed values
  float* qs = vv + kSimtTT * D;            // [G][D]
  float* pp = qs + G * D;                  // [G][TT]   logits, then probabilities
  __shared__ int s_cid[kSimtTT];
  __shared__ int s_pos[kSimtTT];    // row of the token in the cache (-1: none)
  __shared__ int s_rpos[kSimtTT];   // its RoPE position (the original one after eviction)
  __shared__ float s_ml[kMaxG][2];

  if (tid < CPT) {
    const int slot = tile * CPT + tid;
    int c = slot < k ? a.sel[(size_t)p * k + slot] : -1;
    if (c >= dm.Nc) { raise_status(a.status, kStatusDeviceCheck); c = -1; }
    s_cid[tid] = c;
  }
  for (int i = tid; i < G * D; i += blockDim.x)
    qs[i] = ldf((const T*)a.q, ((size_t)b * dm.Hq + (size_t)h * G) * D + i);
  __syncthreads();
  if (tid < kSimtTT) {
    const int c = s_cid[tid / C];
    s_pos[tid] = c >= 0 ? c * C + tid % C : -1;
    s_rpos[tid] = c >= 0 ? chunk_position(dm, a.chunk_pos, b, c, a.status) * C + tid % C : -1;
  }
  __syncthreads();

  // coefficients of the tile's tokens
  const T* coef = (const T*)a.coef;
  for (int i = tid; i < kSimtTT * r; i += blockDim.x) {
    const int t = i / r, kk = i - t * r;
    const int pos = s_pos[t];
    cs[i] = pos >= 0 ? ldf(coef, ((size_t)b * dm.T + pos) * r + kk) : 0.f;
  }
  __syncthreads();

  // K~_pre = B_h c
  {
    constexpr int NG = kSimtThreads / D;
    constexpr int R = kSimtTT / NG;
    const int j = tid % D, tg = tid / D;
    const T* brow = (const T*)a.basis + ((size_t)h * D + j) * r;
    float acc[R];
#pragma unroll
    for (int i = 0; i < R; ++i) acc[i] = 0.f;
    for (int kk = 0; kk < r; ++kk) {
      const float bj = ldf(brow, kk);
#pragma unroll
      for (int i = 0; i < R; ++i) acc[i] = fmaf(bj, cs[(tg + NG * i) * r + kk], acc[i]);
    }
#pragma unroll
    for (int i = 0; i < R; ++i) kp[(tg + NG * i) * D + j] = acc[i];
  }
  __syncthreads();

  // logits z_g,t = q_g . R(t) K~_pre,t / sqrt(d): 8 threads per token, split over pairs
  {
    const int t = tid >> 3, part = tid & 7;
    const int pos = s_pos[t];
    float acc[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) acc[g] = 0.f;
    if (pos >= 0) {
      for (int i = part; i < D / 2; i += 8) {
        const float2 cs2 = rope_cs32(a.rope, i, s_rpos[t]);
        const float x = kp[t * D + i], y = kp[t * D + i + D / 2];
        const float xr = x * cs2.x - y * cs2.y;
        const float yr = x * cs2.y + y * cs2.x;
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < G) acc[g] = fmaf(qs[g * D + i], xr, fmaf(qs[g * D + i + D / 2], yr, acc[g]));
      }
    }
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      float v = acc[g];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      acc[g] = v;
    }
    if (part == 0) {
      const float scale = rsqrtf((float)D);
      for (int g = 0; g < G; ++g) pp[g * kSimtTT + t] = pos >= 0 ? acc[g] * scale : -INFINITY;
    }
  }

  // hidden = act(W1 K~_pre + b1)
  {
    constexpr int NG = kSimtThreads / FH;
    constexpr int R = kSimtTT / NG;
    const int f = tid % FH, tg = tid / FH;
    const T* wrow = (const T*)a.w1 + ((size_t)h * FH + f) * D;
    float acc[R];
#pragma unroll
    for (int i = 0; i < R; ++i) acc[i] = 0.f;
    for (int j = 0; j < D; ++j) {
      const float w = ldf(wrow, j);
#pragma unroll
      for (int i = 0; i < R; ++i) acc[i] = fmaf(w, kp[(tg + NG * i) * D + j], acc[i]);
    }
    const float bias = ldf((const T*)a.b1, (size_t)h * FH + f);
#pragma unroll
    for (int i = 0; i < R; ++i) hid[(tg + NG * i) * FH + f] = act_f(acc[i] + bias, dm.act);
  }
  __syncthreads();

  // V~ = W2 hidden + b2
  {
    constexpr int NG = kSimtThreads / D;
    constexpr int R = kSimtTT / NG;
    const int j = tid % D, tg = tid / D;
    const T* wrow = (const T*)a.w2 + ((size_t)h * D + j) * FH;
    float acc[R];
#pragma unroll
    for (int i = 0; i < R; ++i) acc[i] = 0.f;
    for (int f = 0; f < FH; ++f) {
      const float w = ldf(wrow, f);
#pragma unroll
      for (int i = 0; i < R; ++i) acc[i] = fmaf(w, hid[(tg + NG * i) * FH + f], acc[i]);
    }
    const float bias = ldf((const T*)a.b2, (size_t)h * D + j);
#pragma unroll
    for (int i = 0; i < R; ++i) vv[(tg + NG * i) * D + j] = acc[i] + bias;
  }
  __syncthreads();

  // residual corrections of the tile's chunks (CSR spans; every index bounds-checked)
  {
    constexpr int NG = kSimtThreads / D;
    const int j = tid % D, tg = tid / D;
    const int32_t* ptr = a.chunk_ptr + (size_t)p * (dm.Nc + 1);
    const int32_t* ridx = a.res_idx + (size_t)p * dm.n_res;
    const T* rval = (const T*)a.res_val + (size_t)p * dm.n_res * D;
    for (int slot = tg; slot < CPT; slot += NG) {
      const int c = s_cid[slot];
      if (c < 0) continue;
      const int e0 = ptr[c], e1 = ptr[c + 1];
      if (e0 < 0 || e1 < e0 || e1 > dm.n_res || e1 - e0 > C) {
        if (j == 0) raise_status(a.status, kStatusDeviceCheck);
        continue;
      }
      for (int e = e0; e < e1; ++e) {
        const int t = ridx[e] - c * C;
        if (t < 0 || t >= C) {
          if (j == 0) raise_status(a.status, kStatusDeviceCheck);
          continue;
        }
        vv[(slot * C + t) * D + j] +=
            dm.res_int4 ? int4_residual((const uint8_t*)a.res_val, (const __half*)a.res_scale, dm,
                                        (size_t)p * dm.n_res + e, j)
                        : ldf(rval, (size_t)e * D + j);
      }
    }
  }
  __syncthreads();

  // tile softmax statistics (warp per query head; one lane per token)
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int g = warp; g < G; g += kSimtThreads / 32) {
      const float z = pp[g * kSimtTT + lane];
      const float m = warp_max(z);
      const float e = (m == -INFINITY) ? 0.f : expf(z - m);
      const float l = warp_sum(e);
      pp[g * kSimtTT + lane] = e;
      if (lane == 0) { s_ml[g][0] = m; s_ml[g][1] = l; }
    }
  }
  __syncthreads();

  // partial: [g][m, l, acc[D]] with acc = sum_t e_t V~_t
  float* part = a.part + ((size_t)p * a.n_tiles + tile) * (size_t)G * (2 + D);
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int g = i / D, j = i - g * D;
    float acc = 0.f;
#pragma unroll 8
    for (int t = 0; t < kSimtTT; ++t) acc = fmaf(pp[g * kSimtTT + t], vv[t * D + j], acc);
    part[g * (2 + D) + 2 + j] = acc;
  }
  if (tid < G) {
    part[tid * (2 + D)] = s_ml[tid][0];
    part[tid * (2 + D) + 1] = s_ml[tid][1];
  }
}

// Combine, plain form: out_g = sum_tiles e^{m_t - M} acc_t / sum_tiles e^{m_t - M} l_t.
template <typename T, int D>
__global__ void __launch_bounds__(256) combine_plain_kernel(const AttendArgs a) {
  const Dims& dm = a.dm;
  const int p = blockIdx.x, b = p / dm.H, h = p % dm.H, G = dm.G;
  const float* part = a.part + (size_t)p * a.n_tiles * G * (2 + D);
  const size_t tstride = (size_t)G * (2 + D);
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int g = i / D, j = i - g * D;
    float M = -INFINITY;
#pragma unroll 8
    for (int t = 0; t < a.n_tiles; ++t) M = fmaxf(M, part[t * tstride + g * (2 + D)]);
    float L = 0.f, O = 0.f;
#pragma unroll 8
    for (int t = 0; t < a.n_tiles; ++t) {
      const float* pt = part + t * tstride + g * (2 + D);
      const float w = pt[0] == -INFINITY ? 0.f : expf(pt[0] - M);
      L = fmaf(w, pt[1], L);
      O = fmaf(w, pt[2 + j], O);
    }
    const size_t oi = ((size_t)b * dm.Hq + (size_t)h * G + g) * D + j;
    if (a.out_f32) {   // decode with a suffix: the merge kernel finishes the output
      a.out_f32[oi] = O / L;
      if (j == 0) {
        a.out_ml[2 * (oi / D)] = M;
        a.out_ml[2 * (oi / D) + 1] = L;
      }
    } else {
      ((T*)a.out)[oi] = from_f<T>(O / L);
    }
  }
}

// Combine, W2-after-attention form used by the tensor-core kernel. Partial of a tile:
// [G][2] (m in log2 units, l), [G][F] sum_t e_t act(h_t), [2][G][D] sum_t e_t R_t.
//   out_g = (W2 Hs_g + Rs_g) / L_g + b2,   Hs/Rs/L the 2^(m_t-M)-weighted tile sums.
// One CTA per (b, h, g); n_tiles <= 64 (checked on the host). Every global load of a
// thread is issued before the arithmetic that needs it: the kernel is a few round trips.
template <typename T, int D, int FH>
__global__ void __launch_bounds__(256) combine_reorder_kernel(const AttendArgs a) {
  static_assert(FH == 256 && D == 128, "combine shape");
  const Dims& dm = a.dm;
  const int G = dm.G;
  const int p = blockIdx.x / G, g = blockIdx.x % G;
  const int b = p / dm.H, h = p % dm.H;
  const int n = a.n_tiles;
  const size_t tstride = (size_t)G * 2 + (size_t)G * FH + (size_t)kTcResSlots * G * D;
  const float* part = a.part + (size_t)p * n * tstride;
  __shared__ float hs[FH];
  __shared__ float rs[2][D];
  __shared__ float s_L;
  const int tid = threadIdx.x, lane = tid & 31;
  // this thread's output row j = tid / 2, half of F: 128 bf16 of W2, loaded now
  const int j = tid >> 1, half = tid & 1;
  uint4 w2v[FH / 2 / 8];
  {
    const uint4* wrow = reinterpret_cast<const uint4*>(
        (const T*)a.w2 + ((size_t)h * D + j) * FH + half * (FH / 2));
#pragma unroll
    for (int i = 0; i < FH / 2 / 8; ++i) w2v[i] = wrow[i];
  }
  // launched as a programmatic dependent of the attend kernel: W2 above is independent
  // of it; the partials, flags and counters below are not
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (a.ready && g == 0 && threadIdx.x == 0 && (b & 31) == 0)   // the next step's words
    a.ready[ready_word(dm, b, h)] = 0;
  if (a.item_ctr && p < dm.H && g == 0 && threadIdx.x == 0) a.item_ctr[p] = 0;   // tile counters
  const float b2 = ldf((const T*)a.b2, (size_t)h * D + j);
  // tile weights, computed by every warp: lane t holds tile t (and t + 32)
  const float m0 = lane < n ? part[lane * tstride + 2 * g] : -INFINITY;
  const float m1 = lane + 32 < n ? part[(lane + 32) * tstride + 2 * g] : -INFINITY;
  const float l0 = lane < n ? part[lane * tstride + 2 * g + 1] : 0.f;
  const float l1 = lane + 32 < n ? part[(lane + 32) * tstride + 2 * g + 1] : 0.f;
  const float* hsrc = part + 2 * G + (size_t)g * FH + tid;                       // f = tid
  const float* rsrc = part + 2 * G + (size_t)G * FH + (size_t)(tid >> 7) * G * D + (size_t)g * D + (tid & 127);
  float hacc = 0.f, racc = 0.f;
  const float M = warp_max(fmaxf(m0, m1));
  const float w0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M);
  const float w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
  for (int t0 = 0; t0 < n; t0 += 16) {
    float hv[16], rv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int t = t0 + u;
      hv[u] = t < n ? hsrc[t * tstride] : 0.f;
      // this thread sums residual slots (tid >> 7), (tid >> 7) + 2, ...
      float r = 0.f;
      if (t < n)
        for (int sl = 0; sl + (tid >> 7) < kTcResSlots; sl += 2) r += rsrc[t * tstride + (size_t)sl * G * D];
      rv[u] = r;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int t = t0 + u;
      const float wt = __shfl_sync(0xffffffffu, t < 32 ? w0 : w1, t & 31);
      hacc = fmaf(wt, hv[u], hacc);
      racc = fmaf(wt, rv[u], racc);
    }
  }
  const float L = warp_sum(w0 * l0 + w1 * l1);
  hs[tid] = hacc;
  rs[tid >> 7][tid & 127] = racc;
  if (tid == 0) s_L = L;
  __syncthreads();
  float acc = 0.f;
  const float* hh = hs + half * (FH / 2);
#pragma unroll
  for (int i = 0; i < FH / 2 / 8; ++i) {
    float w[8];
    const uint4 v = w2v[i];
    if constexpr (sizeof(T) == 2) {
      const float2 a0 = bf2_to_f2(v.x), a1 = bf2_to_f2(v.y), a2 = bf2_to_f2(v.z), a3 = bf2_to_f2(v.w);
      w[0] = a0.x; w[1] = a0.y; w[2] = a1.x; w[3] = a1.y; w[4] = a2.x; w[5] = a2.y; w[6] = a3.x; w[7] = a3.y;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(w[e], hh[8 * i + e], acc);
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  if (half == 0) {
    const size_t oi = ((size_t)b * dm.Hq + (size_t)h * G + g) * D + j;
    const float o = (acc + rs[0][j] + rs[1][j]) / s_L + b2;
    if (a.out_f32) {   // decode with a suffix: max in natural-log units, and the sum
      a.out_f32[oi] = o;
      if (j == 0) {
        a.out_ml[2 * (oi / D)] = M * 0.69314718055994531f;
        a.out_ml[2 * (oi / D) + 1] = s_L;
      }
    } else {
      ((T*)a.out)[oi] = from_f<T>(o);
    }
  }
}

template <typename T, int D, int FH>
cudaError_t launch_simt_typed(const AttendArgs& a, cudaStream_t s) {
  const size_t smem = SimtSmem<D, FH>::floats(a.dm.r, a.dm.G) * sizeof(float);
  auto kern = attend_simt_kernel<T, D, FH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_tiles, a.dm.B * a.dm.H);
  kern<<<grid, kSimtThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

int attend_simt_tile_tokens(const Dims&) { return kSimtTT; }

size_t attend_simt_part_floats(const Dims& dm, int n_tiles) {
  return (size_t)dm.B * dm.H * n_tiles * dm.G * (2 + dm.d);
}

cudaError_t launch_attend_simt(const AttendArgs& a, cudaStream_t s) {
  const bool bf = a.dm.dtype == LOWRAM_DTYPE_BF16;
  const int D = a.dm.d, FH = a.dm.F;
#define LR_CASE(DD, FF)                                                      \
  if (D == DD && FH == FF)                                                   \
    return bf ? launch_simt_typed<__nv_bfloat16, DD, FF>(a, s)               \
              : launch_simt_typed<float, DD, FF>(a, s);
  LR_CASE(64, 128) LR_CASE(64, 256) LR_CASE(128, 128) LR_CASE(128, 256)
#undef LR_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(const AttendArgs& a, bool reorder_form, cudaStream_t s) {
  const bool bf = a.dm.dtype == LOWRAM_DTYPE_BF16;
  const int D = a.dm.d, FH = a.dm.F;
  const int grid = a.dm.B * a.dm.H;
  if (!reorder_form) {
    if (D == 64) {
      if (bf) combine_plain_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(a);
      else combine_plain_kernel<float, 64><<<grid, 256, 0, s>>>(a);
    } else if (D == 128) {
      if (bf) combine_plain_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(a);
      else combine_plain_kernel<float, 128><<<grid, 256, 0, s>>>(a);
    } else {
      return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
  }
  if (D == 128 && FH == 256 && bf) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid * a.dm.G);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, combine_reorder_kernel<__nv_bfloat16, 128, 256>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  return cudaErrorInvalidValue;
}

}  // namespace lowram
