// Uncompressed GQA flash-decode over a bf16 KV cache: the baseline that LowRAM's
// compressed decode is compared against (the pages compare decode throughput with the
// uncompressed model and report about five times its peak decode throughput at 262K
// tokens: agihunt summary, efficiency paragraph; cctest "How the method works",
// Selective reconstruction; the abstract).
//
//   out_g = sum_t softmax_t(q_g . K_t / sqrt(d)) V_t over every position t < T, for each
//   query head g of the KV head's GQA group (the oracle's dense_attention).
//
// HBM-bound (every K and V byte is read once, ~4 FLOP per byte): CUDA cores, no tensor
// cores. Split-K: a CTA takes 1024 positions of one (b, h). Its K and V rows arrive by
// TMA in tiles of 64 positions (one 64 x 128 box of each, 32 KB) into a 3-stage ring,
// so the loads stay in flight while the warps compute; one elected thread refills a
// stage once all eight warps have released it. In a tile, warp w takes positions
// 8w .. 8w + 7; 16 lanes hold one position's row (8 dimensions each, one 16-byte
// shared-memory load); every lane group takes four positions, reduces their 16 logits
// with one reduce-scatter (15 shuffles), updates the online softmax once, and accumulates
// V. The CTA's partial (m, l, O) goes to the workspace; a combine kernel merges the
// splits of each query head. Every wait is bounded; on expiry the kernel raises a
// timeout status, lets its copies in flight land and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace lowram {
namespace {

using namespace sm100;

constexpr int kDD = 128, kDG = 4;
constexpr int kDenseThreads = 256;
constexpr int kDenseSplit = 1024;   // positions per CTA
constexpr int kPartStride = kDG * (2 + kDD);
constexpr int kTilePos = 64;                             // positions per TMA tile
constexpr int kDStages = 3;                              // ring depth
constexpr uint32_t kRowBytes = kDD * 2;                  // one head's row, bf16
constexpr uint32_t kHalfBytes = kTilePos * kRowBytes;    // K (or V) of one tile: 16 KB
constexpr uint32_t kStageBytes = 2 * kHalfBytes;
constexpr size_t kDenseSmem = (size_t)kDStages * kStageBytes + 128 + 128;   // + barriers + align
static_assert(kDenseSplit % kTilePos == 0 && kTilePos == 8 * (kDenseThreads / 32),
              "a tile gives each warp 8 positions");

struct DenseMaps {
  CUtensorMap k;   // [B*T rows][H*d cols] bf16, box 128 x 64
  CUtensorMap v;
};

struct DenseArgs {
  int B, T, H, Hq;
  const __nv_bfloat16* k;   // [B][T][H][d]
  const __nv_bfloat16* v;   // [B][T][H][d]
  const __nv_bfloat16* q;   // [B][Hq][d]
  __nv_bfloat16* out;       // [B][Hq][d]
  float* part;              // [B*H][n_split][G][2 + d]
  int n_split;
  int t_valid;              // positions 0 .. t_valid-1 of each row block are attended
  int* status;              // device status word (timeout)
};

__global__ void __launch_bounds__(kDenseThreads, 2)
dense_decode_kernel(const DenseArgs a, const __grid_constant__ DenseMaps maps) {
  const int p = blockIdx.y, b = p / a.H, h = p % a.H;
  const int split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 4, gl = lane & 15;
  const int t_begin = split * kDenseSplit;
  const int t_end = min(a.t_valid, t_begin + kDenseSplit);
  const int n_tiles = (t_end - t_begin + kTilePos - 1) / kTilePos;
  extern __shared__ uint8_t dsm_raw[];
  const uint32_t raw = smem_u32(dsm_raw);
  const uint32_t ring = (raw + 127u) & ~127u;
  uint8_t* gring = dsm_raw + (ring - raw);
  const uint32_t bars = ring + kDStages * kStageBytes;   // full[kDStages], empty[kDStages]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gring + kDStages * kStageBytes + 64);
  auto full = [&](int st) { return bars + 8u * (uint32_t)st; };
  auto empty = [&](int st) { return bars + 8u * (uint32_t)(kDStages + st); };
  // tile j: positions t_begin + 64 j .., rows b T + t of the [B*T][H*d] view, columns h d ..
  auto issue = [&](int j) {
    const int st = j % kDStages;
    const uint32_t dst = ring + (uint32_t)st * kStageBytes;
    mbar_arrive_expect_tx(full(st), kStageBytes);
    const int y = b * a.T + t_begin + kTilePos * j;
    tma_load_2d(dst, &maps.k, h * kDD, y, full(st));
    tma_load_2d(dst + kHalfBytes, &maps.v, h * kDD, y, full(st));
  };
  if (tid == 0) {
    *abort_flag = 0;
    for (int st = 0; st < kDStages; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), kDenseThreads / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();
  int issued = 0, landed = 0;   // thread 0: tiles requested / seen complete (for the drain)
  if (tid == 0)
    for (; issued < kDStages && issued < n_tiles; ++issued) issue(issued);
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
  // in tile j, lane group grp of warp w takes positions 8 w + 4 grp + u (u < 4)
  bool good = true;
#pragma unroll 1
  for (int i = 0; i < n_tiles; ++i) {
    const int st = i % kDStages;
    good = good && mbar_wait_bounded(full(st), (uint32_t)((i / kDStages) & 1), abort_flag);
    if (tid == 0 && good) landed = i + 1;
    const int pl0 = 8 * warp + 4 * grp;                  // first position of the lane group
    const int w0 = t_begin + kTilePos * i + pl0;
    const uint8_t* kst = gring + st * kStageBytes + (size_t)pl0 * kRowBytes + 16 * gl;
    uint4 kr[4], vr[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      kr[u] = *reinterpret_cast<const uint4*>(kst + u * kRowBytes);
      vr[u] = *reinterpret_cast<const uint4*>(kst + kHalfBytes + u * kRowBytes);
    }
    // the stage may be refilled once every warp has its rows in registers
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
    if (tid == 0 && i + kDStages < n_tiles) {
      good = good && mbar_wait_bounded(empty(st), (uint32_t)((i / kDStages) & 1), abort_flag);
      if (good) issue(issued++);
    }
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
    const bool valid = good && w0 + my_u < t_end;
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
  if (tid == 0 && *abort_flag) {   // a wait gave up: the copies still in flight land first
    raise_status(a.status, kStatusTimeout);
    for (int j = landed; j < issued; ++j) {
      int dummy = 0;
      mbar_wait_bounded(full(j % kDStages), (uint32_t)((j / kDStages) & 1), (volatile int*)&dummy);
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

// The split kernel over a.n_split x (B*H) CTAs: tensor maps over the [B*T][H*d] views of
// K and V (one head's 64 x 128 box per tile), then the launch.
cudaError_t launch_splits(const DenseArgs& a, cudaStream_t s) {
  DenseMaps maps;
  const uint64_t rows = (uint64_t)a.B * a.T, cols = (uint64_t)a.H * kDD;
  if (!make_tensor_map_2d(&maps.k, a.k, LOWRAM_DTYPE_BF16, cols, rows, kDD, kTilePos, 0, 256) ||
      !make_tensor_map_2d(&maps.v, a.v, LOWRAM_DTYPE_BF16, cols, rows, kDD, kTilePos, 0, 256))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(dense_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kDenseSmem);
  if (e != cudaSuccess) return e;
  dense_decode_kernel<<<dim3(a.n_split, a.B * a.H), kDenseThreads, kDenseSmem, s>>>(a, maps);
  return cudaGetLastError();
}

}  // namespace

size_t suffix_workspace_bytes(const Dims& dm, int s_max) {
  const size_t n_split = (size_t)(s_max + kDenseSplit - 1) / kDenseSplit;
  return (size_t)dm.B * dm.H * (n_split > 0 ? n_split : 1) * kPartStride * sizeof(float);
}

cudaError_t launch_suffix_merge(const Dims& dm, const void* k_suffix, const void* v_suffix,
                                int s_max, int n_suffix, const void* q, const float* pre_out,
                                const float* pre_ml, void* out, void* ws, int* status,
                                cudaStream_t s) {
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
  a.status = status;
  a.n_split = (n_suffix + kDenseSplit - 1) / kDenseSplit;
  if (a.n_split > 0) {
    const cudaError_t e = launch_splits(a, s);
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
                                void* out, void* ws, int* status, cudaStream_t s) {
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
  a.status = status;
  cudaError_t e = launch_splits(a, s);
  if (e != cudaSuccess) return e;
  dense_combine_kernel<<<dm.B * dm.Hq, kDD, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace lowram
