// Kernel (c), tensor-core form: the encode's contractions on tcgen05 / TMEM (bf16 storage,
// d = 128, F = 256, r % 32 == 0, 32 <= r <= 160, T % 128 == 0).
//
// Method (LowRAM summary on agihunt.info, key paragraph: RoPE is inverted and the keys
// are projected onto the xKV basis; value-cache-amortisation paragraph and cctest "How
// the method works": Amortised values, Residuals for difficult tokens):
//   project kernel (E1, E2): per tile of 128 tokens, c = K_pre B over D = H_kv d, where
//     K_pre is the inverse-rotated key of every head: an MMA with M = 128 tokens, N = r,
//     K = D, accumulated in Tensor Memory over the heads. It stores c unrounded (fp32, in
//     the workspace) and rounded (the cache's coef).
//   predict kernel (E4 / E6): per (tile of 128 tokens, KV head h), the predictor chain
//     as three MMAs: K~ = c B_h^T (N = d, K = r), H = K~ W1_h^T (N = F, K = d),
//     V_hat = act(H + b1) W2_h^T (N = d, K = F); then the squared error
//     e_t = |V_t - V_hat_t - b2|^2 of every token (with the unrounded c), or, for the
//     picked tokens, the residual row R_t = V_t - V_hat_t - b2 (with the stored coef).
//
// Precision. Each operand that is not a stored bf16 value (K_pre, c, K~, act) enters
// its MMA as two bf16 terms, x = hi + lo with hi = bf16(x) and lo = bf16(x - hi)
// (x - hi is exact in fp32), so it carries about 16 significant bits; the weights and
// the basis are stored bf16 values and enter exactly. Products of bf16 values are exact
// and accumulate in fp32. The errors come out within ~1e-4 relative, inside the window
// around the selection threshold that the residual pick re-scores in fp64.
//
// Shared-memory operands are K-major with the 64-byte swizzle in blocks of 32 columns
// ([rows][64 B] per block): the A operands are written by threads, the B operands
// (basis, W1, W2) are TMA tiles of the same form.
// Every wait is bounded (~2 s); on expiry the kernel raises a timeout status, drains its
// outstanding copies and MMAs (bounded), frees Tensor Memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace lowram {
namespace {

using namespace sm100;

constexpr int kD = 128, kF = 256, kM = 128;
constexpr int kThreads = 256;   // 8 warps: two per Tensor Memory lane quadrant
constexpr uint32_t kBlk = 8192; // one [128 rows][32 columns] bf16 block (64 B rows)

// x = hi + lo for two consecutive values, packed as bf16 pairs (first value low).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x0, x1);
  const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
  lo = pack_bf16x2(x0 - h0, x1 - h1);
}

// Store 8 consecutive fp32 values (columns 8*cc .. 8*cc+7 of row `row`) of an A operand as
// hi and lo bf16 blocks: block cc / 4, 16-byte chunk cc % 4, 64-byte swizzle.
__device__ __forceinline__ void store_split8(uint32_t hi_base, uint32_t lo_base, int row,
                                             int cc, const float* v) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) split2(v[2 * i], v[2 * i + 1], h[i], l[i]);
  const uint32_t off = (uint32_t)(cc >> 2) * kBlk + sw64_offset(row, cc & 3);
  st_shared_v4(hi_base + off, h[0], h[1], h[2], h[3]);
  st_shared_v4(lo_base + off, l[0], l[1], l[2], l[3]);
}

// K-step s (16 columns) of a 64B-swizzled K-major operand whose 32-column blocks are
// `blk` bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int s, uint32_t blk) {
  return smem_desc_kmajor(base + (uint32_t)(s >> 1) * blk + (uint32_t)(s & 1) * 32u, 512,
                          kSwizzle64B);
}

// The activation between the hidden and the output MMA: SiLU as x / (1 + e^-x) with the
// fast exponential and division (relative error ~1e-6, far inside what the errors' fp64
// re-scoring window allows); erf-GELU with erff.
__device__ __forceinline__ float act_acc(float x, int act) {
  if (act == LOWRAM_ACT_SILU) return __fdividef(x, 1.0f + __expf(-x));
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

// ---------------------------------------------------------------- project kernel
struct ProjMaps {
  CUtensorMap basis_t;   // [r][D] bf16 (the basis transposed), box 32 x r, 64B swizzle
};

// smem: A[2] (hi 32 KB + lo 32 KB each), Bt[2] (r x 256 B each), barriers
__host__ __device__ inline uint32_t proj_smem_bytes(int r) {
  return 2 * 65536u + 2u * (uint32_t)r * 256u + 1024u + 1024u;
}

__global__ void __launch_bounds__(kThreads, 1)
encode_project_tc_kernel(const EncodeArgs a, const __grid_constant__ ProjMaps maps,
                         float* c_ws) {
  const Dims& dm = a.dm;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int r = dm.r, H = dm.H;
  const uint32_t sA = base, sB = base + 2 * 65536u;
  const uint32_t bt_bytes = (uint32_t)r * 256u;
  const uint32_t sBar = sB + 2 * bt_bytes;
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };   // 0,1 full; 2,3 empty; 4 done; 5 drain
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + (sBar - base) + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + (sBar - base) + 68);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 6; ++i) mbar_init(bar(i), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t idesc = idesc_bf16_f32(kM, r);
  const int tiles_per_b = dm.T / kM;
  const int n_tiles = dm.B * tiles_per_b;
  const int row = tid & (kM - 1), hf = tid >> 7;
  const __nv_bfloat16* kc = (const __nv_bfloat16*)a.k_cache;
  int n_issued = 0;   // head passes issued by this CTA (TMA + MMA), for the parities

  int it = 0;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
    const int b = tile / tiles_per_b, t0 = (tile % tiles_per_b) * kM;
    const int t = t0 + row;
    const int pos = token_position(dm, a.chunk_pos, b, t, a.status);   // RoPE position
    // the token's rotations (cos, sin)(pos theta_i) of this thread's 32 pairs, shared by
    // all heads; and head 0's key rows
    float2 rc[32];
    {   // 16-byte loads of both tables' rows (pairs 32 hf .. 32 hf + 31 are contiguous)
      const float4* lo4 = reinterpret_cast<const float4*>(
          a.rope.lo32 + (size_t)(pos & (kRopeLo - 1)) * a.rope.half + 32 * hf);
      const float4* hi4 = reinterpret_cast<const float4*>(
          a.rope.hi32 + (size_t)(pos >> kRopeLoBits) * a.rope.half + 32 * hf);
#pragma unroll
      for (int m8 = 0; m8 < 16; m8 += 8) {
        float4 lv[8], hv[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          lv[m] = __ldg(lo4 + m8 + m);
          hv[m] = __ldg(hi4 + m8 + m);
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          rc[2 * (m8 + m)] = rope_combine(make_float2(hv[m].x, hv[m].y), make_float2(lv[m].x, lv[m].y));
          rc[2 * (m8 + m) + 1] =
              rope_combine(make_float2(hv[m].z, hv[m].w), make_float2(lv[m].z, lv[m].w));
        }
      }
    }
    const __nv_bfloat16* src0 = kc + ((size_t)b * dm.T + t) * H * kD + 32 * hf;
    uint4 xr[4], yr[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      xr[q] = *reinterpret_cast<const uint4*>(src0 + 8 * q);
      yr[q] = *reinterpret_cast<const uint4*>(src0 + kD / 2 + 8 * q);
    }
    for (int h = 0; h < H; ++h) {
      const int n = it * H + h, u = n & 1, j = n >> 1;
      // buffer u is free once the MMAs of pass n - 2 have completed
      mbar_wait_bounded(bar(2 + u), (uint32_t)((j & 1) ^ 1), abort_flag);
      if (tid == 0) {
        mbar_arrive_expect_tx(bar(u), 4u * (uint32_t)r * 64u);
        for (int kb = 0; kb < 4; ++kb)
          tma_load_2d(sB + (uint32_t)u * bt_bytes + (uint32_t)kb * (uint32_t)r * 64u,
                      &maps.basis_t, h * kD + kb * 32, 0, bar(u));
      }
      // E1: K_pre = R(t)^T K of head h for pairs i = 32 hf .. 32 hf + 31 of this token;
      // the next head's rows are loaded first, so their latency hides behind this head
      uint4 xn[4], yn[4];
      if (h + 1 < H) {
        const __nv_bfloat16* src = src0 + (size_t)(h + 1) * kD;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          xn[q] = *reinterpret_cast<const uint4*>(src + 8 * q);
          yn[q] = *reinterpret_cast<const uint4*>(src + kD / 2 + 8 * q);
        }
      }
      const uint32_t a_hi = sA + (uint32_t)u * 65536u, a_lo = a_hi + 32768u;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t xw[4] = {xr[q].x, xr[q].y, xr[q].z, xr[q].w};
        const uint32_t yw[4] = {yr[q].x, yr[q].y, yr[q].z, yr[q].w};
        float kx[8], ky[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x2 = bf2_to_f2(xw[e]), y2 = bf2_to_f2(yw[e]);
          const float2 c0 = rc[8 * q + 2 * e], c1 = rc[8 * q + 2 * e + 1];
          kx[2 * e] = x2.x * c0.x + y2.x * c0.y;
          ky[2 * e] = y2.x * c0.x - x2.x * c0.y;
          kx[2 * e + 1] = x2.y * c1.x + y2.y * c1.y;
          ky[2 * e + 1] = y2.y * c1.x - x2.y * c1.y;
        }
        // columns 32 hf + 8 q .. (block hf) and 64 + 32 hf + 8 q .. (block 2 + hf)
        store_split8(a_hi, a_lo, row, 4 * hf + q, kx);
        store_split8(a_hi, a_lo, row, 8 + 4 * hf + q, ky);
      }
      if (h + 1 < H) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          xr[q] = xn[q];
          yr[q] = yn[q];
        }
      }
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        if (mbar_wait_bounded(bar(u), (uint32_t)(j & 1), abort_flag)) {
          tc_fence_after();
          const uint32_t bsm = sB + (uint32_t)u * bt_bytes;
          for (int s = 0; s < kD / 16; ++s) {
            const uint64_t bd = desc_k(bsm, s, (uint32_t)r * 64u);
            mma_bf16(tmem, desc_k(a_hi, s, kBlk), bd, idesc, (h > 0 || s > 0) ? 1u : 0u);
            mma_bf16(tmem, desc_k(a_lo, s, kBlk), bd, idesc, 1u);
          }
        }
        mma_commit(bar(2 + u));
        if (h == H - 1) mma_commit(bar(4));
        ++n_issued;
      }
    }
    // epilogue: c (fp32, unrounded) to the workspace, coef rounded to bf16
    mbar_wait_bounded(bar(4), (uint32_t)(it & 1), abort_flag);
    tc_fence_after();
    {
      const int q = warp & 3, half = warp >> 2;
      const int rr = 32 * q + lane;
      const int ncol = r / 2;
      const size_t tok = (size_t)b * dm.T + t0 + rr;
      float* cdst = c_ws + tok * r + half * ncol;
      __nv_bfloat16* kdst = (__nv_bfloat16*)a.coef + tok * r + half * ncol;
      for (int c0 = 0; c0 < ncol; c0 += 16) {
        float v[16];
        tmem_ld_x16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(half * ncol + c0), v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(cdst + c0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        uint4 w0, w1;
        w0.x = pack_bf16x2(v[0], v[1]); w0.y = pack_bf16x2(v[2], v[3]);
        w0.z = pack_bf16x2(v[4], v[5]); w0.w = pack_bf16x2(v[6], v[7]);
        w1.x = pack_bf16x2(v[8], v[9]); w1.y = pack_bf16x2(v[10], v[11]);
        w1.z = pack_bf16x2(v[12], v[13]); w1.w = pack_bf16x2(v[14], v[15]);
        *reinterpret_cast<uint4*>(kdst + c0) = w0;
        *reinterpret_cast<uint4*>(kdst + c0 + 8) = w1;
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // drain (only needed after an abort): every MMA and copy this CTA issued completes
  if (tid == 0) {
    mma_commit(bar(5));
    int dummy = 0;
    mbar_wait_bounded(bar(5), 0, (volatile int*)&dummy);
    if (*abort_flag) {
      for (int n = n_issued - 2; n < n_issued; ++n) {
        if (n < 0) continue;
        dummy = 0;
        mbar_wait_bounded(bar(n & 1), (uint32_t)((n >> 1) & 1), (volatile int*)&dummy);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) raise_status(a.status, kStatusTimeout);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------- predict kernel
struct PredMaps {
  CUtensorMap basis;   // [H d][r] bf16, box 32 x 128, 64B swizzle
  CUtensorMap w1;      // [H F][d] bf16, box 32 x 256, 64B swizzle
  CUtensorMap w2;      // [H d][F] bf16, box 32 x 128, 64B swizzle
};

// smem: operand A region 128 KB (A1 = c hi/lo, then A2 = K~ hi/lo, then A3 = act hi/lo),
// the basis block of head h right after A1 (r x 256 B), the weight region 64 KB (W1, then
// W2), barriers.
constexpr uint32_t kPredA = 0, kPredW = 131072, kPredBar = 196608;
constexpr uint32_t kPredSmem = kPredBar + 1024 + 1024;   // barriers/part + base alignment

// RES = false: errors e of every token (E4); RES = true: residual rows of the picked
// tokens (E6).
template <bool RES>
__global__ void __launch_bounds__(kThreads, 1)
encode_predict_tc_kernel(const EncodeArgs a, const __grid_constant__ PredMaps maps,
                         const float* c_ws) {
  const Dims& dm = a.dm;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int r = dm.r, H = dm.H;
  const uint32_t sA = base + kPredA, sW = base + kPredW;
  const uint32_t a1_lo = sA + (uint32_t)r * 256u;        // A1 lo after A1 hi (r/32 blocks)
  const uint32_t sB1 = sA + (uint32_t)r * 512u;          // basis_h after A1
  const uint32_t sBar = base + kPredBar;
  // barriers: 0 weights (basis_h + W1), 1 W2, 2 MMA phases, 3 drain
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + kPredBar + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kPredBar + 68);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) mbar_init(bar(i), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tK = tmem, tH = tmem + 128u, tV = tmem + 384u;

  // units: RES = false: (tile of 128 tokens, head), tile-major so that the heads of one
  // tile run close together and share its c rows in L2; RES = true: (pair, 128 picked
  // rows)
  const int tiles_per_b = dm.T / kM;
  const int per_pair = RES ? (dm.n_res + kM - 1) / kM : 0;
  const int n_units = RES ? dm.B * H * per_pair : dm.B * tiles_per_b * H;
  auto unit_of = [&](int u, int& b, int& h, int& r0) {
    if constexpr (RES) {
      const int p = u / per_pair;
      b = p / H;
      h = p % H;
      r0 = (u % per_pair) * kM;
    } else {
      const int tile = u / H;
      h = u % H;
      b = tile / tiles_per_b;
      r0 = (tile % tiles_per_b) * kM;
    }
  };
  // weights of head h for phase 1 and 2 (basis_h, W1_h) on barrier 0
  auto load_w = [&](int h) {
    mbar_arrive_expect_tx(bar(0), (uint32_t)r * 256u + 65536u);
    for (int kb = 0; kb < r / 32; ++kb)
      tma_load_2d(sB1 + (uint32_t)kb * kBlk, &maps.basis, kb * 32, h * kD, bar(0));
    for (int kb = 0; kb < kD / 32; ++kb)
      tma_load_2d(sW + (uint32_t)kb * 16384u, &maps.w1, kb * 32, h * kF, bar(0));
  };
  int loads0 = 0, loads1 = 0, n_mma = 0;
  if (tid == 0 && (int)blockIdx.x < n_units) {
    int b, h, r0;
    unit_of(blockIdx.x, b, h, r0);
    load_w(h);
    ++loads0;
  }
  const int row = tid & (kM - 1), hf = tid >> 7;       // phase-1 role
  const int q = warp & 3, half = warp >> 2;            // Tensor Memory roles
  const int trow = 32 * q + lane;
  const uint32_t lane_addr = (uint32_t)(32 * q) << 16;

  int it = 0;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
    int b, h, r0;
    unit_of(unit, b, h, r0);
    const int p = b * H + h;
    // ---- phase 1: A1 = c rows (split) ----------------------------------------------
    {
      const int ncol = r / 2;
      int tok = -1;
      if (RES) {
        if (r0 + row < dm.n_res) tok = a.res_idx[(size_t)p * dm.n_res + r0 + row];
        if (tok < 0 || tok >= dm.T) tok = -1;
      } else {
        tok = r0 + row;
      }
      for (int c8 = 0; c8 < ncol / 8; ++c8) {
        const int cc = (hf * ncol) / 8 + c8;   // 8-column chunk of the row
        const uint32_t off = (uint32_t)(cc >> 2) * kBlk + sw64_offset(row, cc & 3);
        if (RES) {   // the stored coef is a bf16 value: hi only (lo would be zero)
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (tok >= 0)
            w = *reinterpret_cast<const uint4*>((const __nv_bfloat16*)a.coef +
                                                ((size_t)b * dm.T + tok) * r + 8 * cc);
          st_shared_v4(sA + off, w.x, w.y, w.z, w.w);
        } else {
          const float* src = c_ws + ((size_t)b * dm.T + tok) * r + 8 * cc;
          const float4 v0 = *reinterpret_cast<const float4*>(src);
          const float4 v1 = *reinterpret_cast<const float4*>(src + 4);
          const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          store_split8(sA, a1_lo, row, cc, v);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (mbar_wait_bounded(bar(0), (uint32_t)(it & 1), abort_flag)) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(kM, kD);
        for (int s = 0; s < r / 16; ++s) {
          const uint64_t bd = desc_k(sB1, s, kBlk);
          mma_bf16(tK, desc_k(sA, s, kBlk), bd, idesc, s > 0 ? 1u : 0u);
          if (!RES) mma_bf16(tK, desc_k(a1_lo, s, kBlk), bd, idesc, 1u);
        }
      }
      mma_commit(bar(2));
    }
    mbar_wait_bounded(bar(2), (uint32_t)(n_mma & 1), abort_flag);
    ++n_mma;
    tc_fence_after();
    // ---- phase 2: A2 = K~ (split) ----------------------------------------------------
    {
      const uint32_t a2_lo = sA + 32768u;
#pragma unroll 1
      for (int c32 = 0; c32 < 2; ++c32) {
        float v[32];
        tmem_ld_x32(tK + lane_addr + (uint32_t)(64 * half + 32 * c32), v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) store_split8(sA, a2_lo, trow, 8 * half + 4 * c32 + i, v + 8 * i);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(kM, kF);
      for (int s = 0; s < kD / 16; ++s) {
        const uint64_t bd = desc_k(sW, s, 16384u);
        mma_bf16(tH, desc_k(sA, s, kBlk), bd, idesc, s > 0 ? 1u : 0u);
        mma_bf16(tH, desc_k(sA + 32768u, s, kBlk), bd, idesc, 1u);
      }
      mma_commit(bar(2));
    }
    mbar_wait_bounded(bar(2), (uint32_t)(n_mma & 1), abort_flag);
    ++n_mma;
    tc_fence_after();
    // W1 is consumed: W2_h into the weight region, under the activation work
    if (tid == 0) {
      mbar_arrive_expect_tx(bar(1), 65536u);
      for (int kb = 0; kb < kF / 32; ++kb)
        tma_load_2d(sW + (uint32_t)kb * kBlk, &maps.w2, kb * 32, h * kD, bar(1));
      ++loads1;
    }
    // ---- phase 3: A3 = act(H + b1) (split) -------------------------------------------
    {
      const __nv_bfloat16* b1 = (const __nv_bfloat16*)a.b1 + (size_t)h * kF;
      const uint32_t a3_lo = sA + 65536u;
#pragma unroll 1
      for (int c32 = 0; c32 < 4; ++c32) {
        float v[32];
        tmem_ld_x32(tH + lane_addr + (uint32_t)(128 * half + 32 * c32), v);
        tmem_wait_ld();
        const int f0 = 128 * half + 32 * c32;
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = act_acc(v[e] + __bfloat162float(b1[f0 + e]), dm.act);
#pragma unroll
        for (int i = 0; i < 4; ++i) store_split8(sA, a3_lo, trow, f0 / 8 + i, v + 8 * i);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (mbar_wait_bounded(bar(1), (uint32_t)(it & 1), abort_flag)) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(kM, kD);
        for (int s = 0; s < kF / 16; ++s) {
          const uint64_t bd = desc_k(sW, s, kBlk);
          mma_bf16(tV, desc_k(sA, s, kBlk), bd, idesc, s > 0 ? 1u : 0u);
          mma_bf16(tV, desc_k(sA + 65536u, s, kBlk), bd, idesc, 1u);
        }
      }
      mma_commit(bar(2));
    }
    mbar_wait_bounded(bar(2), (uint32_t)(n_mma & 1), abort_flag);
    ++n_mma;
    tc_fence_after();
    // A3 and W2 are consumed: the next unit's basis_h and W1, under the epilogue
    if (tid == 0 && unit + (int)gridDim.x < n_units) {
      int nb, nh, nr0;
      unit_of(unit + gridDim.x, nb, nh, nr0);
      load_w(nh);
      ++loads0;
    }
    // ---- phase 4: V_hat + b2 against V ----------------------------------------------
    {
      const __nv_bfloat16* b2 = (const __nv_bfloat16*)a.b2 + (size_t)h * kD + 64 * half;
      int tok = -1;
      if (RES) {
        if (r0 + trow < dm.n_res) tok = a.res_idx[(size_t)p * dm.n_res + r0 + trow];
        if (tok < 0 || tok >= dm.T) tok = -1;
      } else {
        tok = r0 + trow;
      }
      const __nv_bfloat16* vsrc =
          (const __nv_bfloat16*)a.v + (((size_t)b * dm.T + (tok < 0 ? 0 : tok)) * H + h) * kD + 64 * half;
      float sq = 0.f;
#pragma unroll 1
      for (int c32 = 0; c32 < 2; ++c32) {
        float v[32];
        tmem_ld_x32(tV + lane_addr + (uint32_t)(64 * half + 32 * c32), v);
        tmem_wait_ld();
        if (tok < 0) continue;
        uint32_t outw[16];
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const uint4 vw = *reinterpret_cast<const uint4*>(vsrc + 32 * c32 + 8 * q8);
          const uint4 bw = *reinterpret_cast<const uint4*>(b2 + 32 * c32 + 8 * q8);
          const uint32_t vv[4] = {vw.x, vw.y, vw.z, vw.w};
          const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 vf = bf2_to_f2(vv[e]), bf = bf2_to_f2(bb[e]);
            const float d0 = vf.x - (v[8 * q8 + 2 * e] + bf.x);
            const float d1 = vf.y - (v[8 * q8 + 2 * e + 1] + bf.y);
            sq = fmaf(d0, d0, fmaf(d1, d1, sq));
            outw[4 * q8 + e] = pack_bf16x2(d0, d1);
          }
        }
        if (RES && dm.res_int4) {
          // the 32 values of this pass are one quantisation group: s = fp16(max|x| / 7),
          // q = clamp(round-half-even(x / s), -8, 7), two codes per byte
          float x[32];
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const uint4 vw = *reinterpret_cast<const uint4*>(vsrc + 32 * c32 + 8 * q8);
            const uint4 bw = *reinterpret_cast<const uint4*>(b2 + 32 * c32 + 8 * q8);
            const uint32_t vv[4] = {vw.x, vw.y, vw.z, vw.w};
            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 vf = bf2_to_f2(vv[e]), bf = bf2_to_f2(bb[e]);
              x[8 * q8 + 2 * e] = vf.x - (v[8 * q8 + 2 * e] + bf.x);
              x[8 * q8 + 2 * e + 1] = vf.y - (v[8 * q8 + 2 * e + 1] + bf.y);
            }
          }
          float amax = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(x[e]));
          const __half sh = __float2half_rn(amax / 7.0f);
          const float sc = __half2float(sh);
          uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            int qv = sc > 0.f ? __float2int_rn(x[e] / sc) : 0;
            qv = qv < -8 ? -8 : (qv > 7 ? 7 : qv);
            words[e >> 3] |= (uint32_t)(qv & 15) << (4 * (e & 7));
          }
          const size_t row = (size_t)p * dm.n_res + r0 + trow;
          const int grp = (64 * half + 32 * c32) / 32;
          *reinterpret_cast<uint4*>((uint8_t*)a.res_val + row * (kD / 2) + 16 * grp) =
              make_uint4(words[0], words[1], words[2], words[3]);
          reinterpret_cast<__half*>(a.res_scale)[row * (kD / 32) + grp] = sh;
        } else if (RES) {
          uint4* dst = reinterpret_cast<uint4*>((__nv_bfloat16*)a.res_val +
                                                ((size_t)p * dm.n_res + r0 + trow) * kD +
                                                64 * half + 32 * c32);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8)
            dst[q8] = make_uint4(outw[4 * q8], outw[4 * q8 + 1], outw[4 * q8 + 2], outw[4 * q8 + 3]);
        }
      }
      if (!RES) {
        // the two column halves of a row meet in shared memory (the barrier slot area
        // holds 128 floats past the barriers)
        float* part = reinterpret_cast<float*>(gbase + kPredBar + 256);
        tc_fence_before();
        __syncthreads();   // the previous unit's readers of `part` are done
        if (half == 1) part[trow] = sq;
        __syncthreads();
        if (half == 0) a.err[(size_t)p * dm.T + tok] = sq + part[trow];
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // drain (only needed after an abort): the weight copies and MMAs this CTA issued
  if (tid == 0) {
    mma_commit(bar(3));
    int dummy = 0;
    mbar_wait_bounded(bar(3), 0, (volatile int*)&dummy);
    if (*abort_flag) {
      if (loads0 > 0) {
        dummy = 0;
        mbar_wait_bounded(bar(0), (uint32_t)((loads0 - 1) & 1), (volatile int*)&dummy);
      }
      if (loads1 > 0) {
        dummy = 0;
        mbar_wait_bounded(bar(1), (uint32_t)((loads1 - 1) & 1), (volatile int*)&dummy);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) raise_status(a.status, kStatusTimeout);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// basis_t[n][k] = basis[k][n] (bf16), the projection MMA's B operand in K-major form.
__global__ void transpose_basis_kernel(const __nv_bfloat16* basis, __nv_bfloat16* basis_t,
                                       int D, int r) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int k0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y)
    if (k0 + i < D && n0 + (int)threadIdx.x < r)
      tile[i][threadIdx.x] = basis[(size_t)(k0 + i) * r + n0 + threadIdx.x];
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y)
    if (n0 + i < r && k0 + (int)threadIdx.x < D)
      basis_t[(size_t)(n0 + i) * D + k0 + threadIdx.x] = tile[threadIdx.x][i];
}

}  // namespace

bool encode_tc_supported(const Dims& dm) {
  return dm.dtype == LOWRAM_DTYPE_BF16 && dm.d == kD && dm.F == kF && dm.r % 32 == 0 &&
         dm.r >= 32 && dm.r <= 160 && dm.T % kM == 0 &&
         (dm.act == LOWRAM_ACT_SILU || dm.act == LOWRAM_ACT_GELU_ERF);
}

cudaError_t launch_encode_project_tc(const EncodeArgs& a, void* basis_t, float* c_ws,
                                     int num_sms, cudaStream_t s) {
  const Dims& dm = a.dm;
  const int D = dm.H * kD;
  dim3 tg((D + 31) / 32, (dm.r + 31) / 32);
  transpose_basis_kernel<<<tg, dim3(32, 8), 0, s>>>((const __nv_bfloat16*)a.basis,
                                                   (__nv_bfloat16*)basis_t, D, dm.r);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ProjMaps maps;
  if (!make_tensor_map_2d(&maps.basis_t, basis_t, LOWRAM_DTYPE_BF16, (uint64_t)D, (uint64_t)dm.r,
                          32, (uint32_t)dm.r, 64))
    return cudaErrorInvalidValue;
  const uint32_t smem = proj_smem_bytes(dm.r);
  if ((e = cudaFuncSetAttribute(encode_project_tc_kernel,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  const int n_tiles = dm.B * (dm.T / kM);
  const int grid = n_tiles < num_sms ? n_tiles : num_sms;
  encode_project_tc_kernel<<<grid, kThreads, smem, s>>>(a, maps, c_ws);
  return cudaGetLastError();
}

cudaError_t launch_encode_predict_tc(const EncodeArgs& a, const float* c_ws, bool residual_rows,
                                     int num_sms, cudaStream_t s) {
  const Dims& dm = a.dm;
  PredMaps maps;
  if (!make_tensor_map_2d(&maps.basis, a.basis, LOWRAM_DTYPE_BF16, dm.r, (uint64_t)dm.H * kD, 32, 128, 64) ||
      !make_tensor_map_2d(&maps.w1, a.w1, LOWRAM_DTYPE_BF16, kD, (uint64_t)dm.H * kF, 32, 256, 64) ||
      !make_tensor_map_2d(&maps.w2, a.w2, LOWRAM_DTYPE_BF16, kF, (uint64_t)dm.H * kD, 32, 128, 64))
    return cudaErrorInvalidValue;
  const int n_units = residual_rows ? dm.B * dm.H * ((dm.n_res + kM - 1) / kM)
                                    : dm.B * (dm.T / kM) * dm.H;
  if (n_units == 0) return cudaSuccess;
  const int grid = n_units < num_sms ? n_units : num_sms;
  auto kern = residual_rows ? encode_predict_tc_kernel<true> : encode_predict_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kPredSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kPredSmem, s>>>(a, maps, c_ws);
  return cudaGetLastError();
}

}  // namespace lowram
