// Uncompressed GQA flash-decode over a bf16 KV cache: the baseline that LowRAM's
// compressed decode is compared against (the pages compare decode throughput with the
// uncompressed model: "up to 5x higher peak decode throughput", agihunt summary,
// efficiency paragraph, and the abstract).
//
//   out_g = sum_t softmax_t(q_g . K_t / sqrt(d)) V_t over every position t < T, for each
//   query head g of the KV head's GQA group (the oracle's dense_attention).
//
// HBM-bound (every K and V byte is read once, ~4 FLOP per byte): CUDA cores, no tensor
// cores. Split-K: a CTA takes 1024 positions of one (b, h); 16 lanes hold one position's
// row (8 dimensions each, so a warp loads two 256-byte rows per instruction); every lane
// group takes four positions per iteration, reduces their 16 logits with one
// reduce-scatter (15 shuffles), updates the online softmax once per four positions, and
// accumulates V. The CTA's partial (m, l, O) goes to the workspace; a combine kernel
// merges the splits of each query head.
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace lowram {
namespace {

constexpr int kDD = 128, kDG = 4;
constexpr int kDenseThreads = 256;
constexpr int kDenseSplit = 1024;   // positions per CTA
constexpr int kPartStride = kDG * (2 + kDD);

struct DenseArgs {
  int B, T, H, Hq;
  const __nv_bfloat16* k;   // [B][T][H][d]
  const __nv_bfloat16* v;   // [B][T][H][d]
  const __nv_bfloat16* q;   // [B][Hq][d]
  __nv_bfloat16* out;       // [B][Hq][d]
  float* part;              // [B*H][n_split][G][2 + d]
  int n_split;
  int t_valid;              // positions 0 .. t_valid-1 of each row block are attended
};

__global__ void __launch_bounds__(kDenseThreads, 2) dense_decode_kernel(const DenseArgs a) {
  const int p = blockIdx.y, b = p / a.H, h = p % a.H;
  const int split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 4, gl = lane & 15;
  const int t_begin = split * kDenseSplit;
  const int t_end = min(a.t_valid, t_begin + kDenseSplit);
  // this lane's 8 dimensions of the group's queries, scaled to log2 units
  const float zs = 1.4426950408889634f * rsqrtf((float)kDD);
  float qv[kDG][8];
#pragma unroll
  for (int g = 0; g < kDG; ++g) {
    const uint4 w = *reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + h * kDG + g) * kDD + 8 * gl);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = bf2_to_f2(ww[e]);
      qv[g][2 * e] = f.x * zs;
      qv[g][2 * e + 1] = f.y * zs;
    }
  }
  float m[kDG], l[kDG], acc[kDG][8];
#pragma unroll
  for (int g = 0; g < kDG; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }
  // positions of this warp: [w0, w0 + 128); lane group grp takes w0 + 8 i + 4 grp + u
  const int w0 = t_begin + warp * (kDenseSplit / (kDenseThreads / 32));
  const size_t row_stride = (size_t)a.H * kDD;
  const __nv_bfloat16* kbase = a.k + ((size_t)b * a.T * a.H + h) * kDD + 8 * gl;
  const __nv_bfloat16* vbase = a.v + ((size_t)b * a.T * a.H + h) * kDD + 8 * gl;
  constexpr int kIters = kDenseSplit / (kDenseThreads / 32) / 8;
  auto load = [&](int i, uint4 (&kk)[4], uint4 (&vv)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = w0 + 8 * i + 4 * grp + u;
      if (t < t_end) {
        kk[u] = __ldcs(reinterpret_cast<const uint4*>(kbase + (size_t)t * row_stride));
        vv[u] = __ldcs(reinterpret_cast<const uint4*>(vbase + (size_t)t * row_stride));
      } else {
        kk[u] = make_uint4(0u, 0u, 0u, 0u);
        vv[u] = kk[u];
      }
    }
  };
#pragma unroll 1
  for (int i = 0; i < kIters; ++i) {
    uint4 kr[4], vr[4];
    load(i, kr, vr);
    // partial logits: z[u][g] over this lane's 8 dimensions
    float z[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t kw[4] = {kr[u].x, kr[u].y, kr[u].z, kr[u].w};
      float kf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = bf2_to_f2(kw[e]);
        kf[2 * e] = f.x;
        kf[2 * e + 1] = f.y;
      }
#pragma unroll
      for (int g = 0; g < kDG; ++g) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) s = fmaf(qv[g][e], kf[e], s);
        z[4 * u + g] = s;
      }
    }
    // reduce-scatter over the 16 lanes: lane gl ends with the full logit of (u, g) =
    // (gl >> 2, gl & 3)
#pragma unroll
    for (int o = 8, n = 16; o >= 1; o >>= 1, n >>= 1) {
      const bool up = (gl & o) != 0;
#pragma unroll
      for (int j = 0; j < n / 2; ++j) {
        const float keep = up ? z[j + n / 2] : z[j];
        const float send = up ? z[j] : z[j + n / 2];
        z[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    const int my_u = gl >> 2, my_g = gl & 3;
    const bool valid = w0 + 8 * i + 4 * grp + my_u < t_end;
    float zz = valid ? z[0] : -INFINITY;
    // block max per head: over the four lanes holding that head's positions
    float bm = fmaxf(zz, __shfl_xor_sync(0xffffffffu, zz, 4));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
    float mnew[kDG], corr[kDG];
#pragma unroll
    for (int g = 0; g < kDG; ++g) {
      const float bg = __shfl_sync(0xffffffffu, bm, (lane & 16) + g);
      mnew[g] = fmaxf(m[g], bg);
      corr[g] = mnew[g] == -INFINITY ? 1.f : exp2f(m[g] - mnew[g]);
    }
    float mine = 0.f;
#pragma unroll
    for (int g = 0; g < kDG; ++g)
      if (my_g == g) mine = valid ? exp2f(zz - mnew[g]) : 0.f;
#pragma unroll
    for (int g = 0; g < kDG; ++g) {
      m[g] = mnew[g];
      l[g] *= corr[g];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] *= corr[g];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t vw[4] = {vr[u].x, vr[u].y, vr[u].z, vr[u].w};
      float vf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = bf2_to_f2(vw[e]);
        vf[2 * e] = f.x;
        vf[2 * e + 1] = f.y;
      }
#pragma unroll
      for (int g = 0; g < kDG; ++g) {
        const float pg = __shfl_sync(0xffffffffu, mine, (lane & 16) + 4 * u + g);
        l[g] += pg;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
      }
    }
  }
  // the two lane groups of the warp, then the warps of the CTA
#pragma unroll
  for (int g = 0; g < kDG; ++g) {
    const float mo = __shfl_xor_sync(0xffffffffu, m[g], 16);
    const float mm = fmaxf(m[g], mo);
    const float c0 = m[g] == -INFINITY ? 0.f : exp2f(m[g] - mm);
    const float c1 = mo == -INFINITY ? 0.f : exp2f(mo - mm);
    l[g] = l[g] * c0 + __shfl_xor_sync(0xffffffffu, l[g], 16) * c1;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      acc[g][e] = acc[g][e] * c0 + __shfl_xor_sync(0xffffffffu, acc[g][e], 16) * c1;
    m[g] = mm;
  }
  __shared__ float s_ml[kDenseThreads / 32][kDG][2];
  __shared__ float s_acc[kDenseThreads / 32][kDG][kDD];
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < kDG; ++g) {
#pragma unroll
      for (int e = 0; e < 8; ++e) s_acc[warp][g][8 * gl + e] = acc[g][e];
      if (gl == 0) {
        s_ml[warp][g][0] = m[g];
        s_ml[warp][g][1] = l[g];
      }
    }
  }
  __syncthreads();
  float* part = a.part + ((size_t)p * a.n_split + split) * kPartStride;
  for (int o = tid; o < kDG * kDD; o += kDenseThreads) {
    const int g = o / kDD, j = o % kDD;
    float M = -INFINITY;
    for (int w = 0; w < kDenseThreads / 32; ++w) M = fmaxf(M, s_ml[w][g][0]);
    float L = 0.f, O = 0.f;
    for (int w = 0; w < kDenseThreads / 32; ++w) {
      const float mw = s_ml[w][g][0];
      const float c = mw == -INFINITY ? 0.f : exp2f(mw - M);
      L = fmaf(c, s_ml[w][g][1], L);
      O = fmaf(c, s_acc[w][g][j], O);
    }
    part[g * (2 + kDD) + 2 + j] = O;
    if (j == 0) {
      part[g * (2 + kDD)] = M;
      part[g * (2 + kDD) + 1] = L;
    }
  }
}

// out_g = sum_s 2^(M_s - M) O_s / sum_s 2^(M_s - M) L_s over the splits s.
__global__ void __launch_bounds__(kDD) dense_combine_kernel(const DenseArgs a) {
  const int bq = blockIdx.x;           // b * Hq + query head
  const int b = bq / a.Hq, hq = bq % a.Hq, h = hq / kDG, g = hq % kDG;
  const int j = threadIdx.x;
  const float* part = a.part + (size_t)(b * a.H + h) * a.n_split * kPartStride + g * (2 + kDD);
  float M = -INFINITY;
  for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, part[(size_t)s * kPartStride]);
  float L = 0.f, O = 0.f;
  for (int s = 0; s < a.n_split; ++s) {
    const float* ps = part + (size_t)s * kPartStride;
    const float c = ps[0] == -INFINITY ? 0.f : exp2f(ps[0] - M);
    L = fmaf(c, ps[1], L);
    O = fmaf(c, ps[2 + j], O);
  }
  a.out[(size_t)bq * kDD + j] = __float2bfloat16_rn(O / L);
}

// Prefix (normalised fp32 output O_c, softmax max M_c in natural-log units and sum L_c)
// merged with the suffix's splits (max in log2 units, sum, unnormalised O):
//   out = (O_c L_c e^(M_c - M) + sum_s O_s e^(M_s - M)) / (L_c e^(M_c - M) + sum_s L_s e^(M_s - M))
__global__ void __launch_bounds__(kDD) suffix_merge_kernel(const DenseArgs a, const float* pre_out,
                                                           const float* pre_ml) {
  const int bq = blockIdx.x;
  const int b = bq / a.Hq, hq = bq % a.Hq, h = hq / kDG, g = hq % kDG;
  const int j = threadIdx.x;
  constexpr float kLn2 = 0.69314718055994531f;
  const float Mc = pre_ml[2 * bq], Lc = pre_ml[2 * bq + 1];
  const float* part = a.part + (size_t)(b * a.H + h) * a.n_split * kPartStride + g * (2 + kDD);
  const int ns = a.t_valid > 0 ? a.n_split : 0;
  float M = Mc;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, part[(size_t)s * kPartStride] * kLn2);
  const float wc = expf(Mc - M);
  float L = Lc * wc, O = pre_out[(size_t)bq * kDD + j] * Lc * wc;
  for (int s = 0; s < ns; ++s) {
    const float* ps = part + (size_t)s * kPartStride;
    const float c = ps[0] == -INFINITY ? 0.f : expf(ps[0] * kLn2 - M);
    L = fmaf(c, ps[1], L);
    O = fmaf(c, ps[2 + j], O);
  }
  a.out[(size_t)bq * kDD + j] = __float2bfloat16_rn(O / L);
}

}  // namespace

size_t suffix_workspace_bytes(const Dims& dm, int s_max) {
  const size_t n_split = (size_t)(s_max + kDenseSplit - 1) / kDenseSplit;
  return (size_t)dm.B * dm.H * (n_split > 0 ? n_split : 1) * kPartStride * sizeof(float);
}

cudaError_t launch_suffix_merge(const Dims& dm, const void* k_suffix, const void* v_suffix,
                                int s_max, int n_suffix, const void* q, const float* pre_out,
                                const float* pre_ml, void* out, void* ws, cudaStream_t s) {
  DenseArgs a{};
  a.B = dm.B;
  a.T = s_max;
  a.H = dm.H;
  a.Hq = dm.Hq;
  a.k = (const __nv_bfloat16*)k_suffix;
  a.v = (const __nv_bfloat16*)v_suffix;
  a.q = (const __nv_bfloat16*)q;
  a.out = (__nv_bfloat16*)out;
  a.part = (float*)ws;
  a.t_valid = n_suffix;
  a.n_split = (n_suffix + kDenseSplit - 1) / kDenseSplit;
  if (a.n_split > 0) {
    dense_decode_kernel<<<dim3(a.n_split, dm.B * dm.H), kDenseThreads, 0, s>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  suffix_merge_kernel<<<dm.B * dm.Hq, kDD, 0, s>>>(a, pre_out, pre_ml);
  return cudaGetLastError();
}

bool dense_supported(const Dims& dm) {
  return dm.dtype == LOWRAM_DTYPE_BF16 && dm.d == kDD && dm.G == kDG;
}

size_t dense_workspace_bytes(const Dims& dm) {
  const size_t n_split = (size_t)(dm.T + kDenseSplit - 1) / kDenseSplit;
  return (size_t)dm.B * dm.H * n_split * kPartStride * sizeof(float);
}

cudaError_t launch_dense_decode(const Dims& dm, const void* k, const void* v, const void* q,
                                void* out, void* ws, cudaStream_t s) {
  DenseArgs a{};
  a.B = dm.B;
  a.T = dm.T;
  a.H = dm.H;
  a.Hq = dm.Hq;
  a.k = (const __nv_bfloat16*)k;
  a.v = (const __nv_bfloat16*)v;
  a.q = (const __nv_bfloat16*)q;
  a.out = (__nv_bfloat16*)out;
  a.part = (float*)ws;
  a.n_split = (dm.T + kDenseSplit - 1) / kDenseSplit;
  a.t_valid = dm.T;
  dense_decode_kernel<<<dim3(a.n_split, dm.B * dm.H), kDenseThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dense_combine_kernel<<<dm.B * dm.Hq, kDD, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace lowram
