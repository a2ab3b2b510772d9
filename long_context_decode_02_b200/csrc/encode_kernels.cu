// Kernel (c): encode one layer's prefix into the compressed cache.
//
// Method (LowRAM summary on agihunt.info, key paragraph: RoPE is inverted before the
// keys are projected onto the xKV basis shared by two adjacent layers, chunk mean keys
// are the landmarks; value-cache-amortisation and ablation paragraphs, cctest "How the
// method works": a per-head key->value predictor, residuals kept only for the
// worst-reconstructed tokens, chosen by error):
//   E1 K_pre = R(t)^T K_cache                      (fp32, host-fp64 RoPE tables)
//   E2 c_t = B^T K_pre,t over D = H_kv*d            -> coef (stored rounded)
//   E3 L_c = mean of the chunk's post-RoPE keys      -> landmark
//   E4 e_t,h = ||V_t,h - MLP_h(B_h c_t)||^2 with the unrounded c (fp32)
//   E5 per (b, h): the n_res largest e (ties -> lower t). fp32 radix select finds the
//      threshold; tokens within 2e-3 relative of it are re-scored with the whole chain
//      recomputed in fp64 and ranked exactly; ascending res_idx and the chunk CSR.
//   E6 R_t = V_t,h - MLP_h(B_h coef_stored,t) for the picked tokens -> res_val
// Encode runs once per prefix; it is not on the per-token decode path.
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace lowram {
namespace {

constexpr int kEncThreads = 256;
constexpr int kTE = 16;          // tokens per CTA in the projection / residual kernels
constexpr int kSelEncThreads = 1024;
constexpr int kRescoreCtas = 96; // CTAs per (b, h) looping over the fp64 candidates
constexpr int kNormRows = 256;   // landmark rows per CTA of the norm bound

// Eight consecutive elements at p (16-byte aligned), read through the read-only path so
// that the loads of a staging loop are issued together rather than one round trip each.
__device__ __forceinline__ void ld8_raw(const __nv_bfloat16* p, __nv_bfloat16 (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  *reinterpret_cast<uint4*>(v) = u;
}
__device__ __forceinline__ void ld8_raw(const float* p, float (&v)[8]) {
  const float4 x = __ldg(reinterpret_cast<const float4*>(p));
  const float4 y = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}

// E3: landmarks, one thread per 8 consecutive output elements (16- or 32-byte loads of
// each of the chunk's C keys, summed in fp32 in token order, then divided by C).
template <typename T>
__global__ void landmark_kernel(const EncodeArgs a) {
  const Dims& dm = a.dm;
  const size_t n8 = (size_t)dm.B * dm.H * dm.Nc * dm.d / 8;
  const T* kc = (const T*)a.k_cache;
  for (size_t o = (size_t)blockIdx.x * blockDim.x + threadIdx.x; o < n8;
       o += (size_t)gridDim.x * blockDim.x) {
    const int j0 = (int)(o % (dm.d / 8)) * 8;
    size_t rest = o / (dm.d / 8);
    const int c = (int)(rest % dm.Nc);
    rest /= dm.Nc;
    const int h = (int)(rest % dm.H);
    const int b = (int)(rest / dm.H);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < dm.C; ++i) {
      T v[8];
      ld8_raw(kc + (((size_t)b * dm.T + (size_t)c * dm.C + i) * dm.H + h) * dm.d + j0, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += to_f(v[e]);
    }
    T out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = from_f<T>(acc[e] / (float)dm.C);
    T* dst = (T*)a.landmark + o * 8;
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(out);
    } else {
      reinterpret_cast<float4*>(dst)[0] = *reinterpret_cast<const float4*>(out);
      reinterpret_cast<float4*>(dst)[1] = *reinterpret_cast<const float4*>(out + 4);
    }
  }
}

// Rebuild keys for kTE tokens and run head h's predictor. cs [kTE][r] holds the
// coefficients; on return vh [kTE][D] holds V_hat. hid is [kTE][FH] scratch.
template <typename T, int D, int FH>
__device__ void predict_tile(const EncodeArgs& a, int h, const float* cs, float* vh,
                             float* hid) {
  const int r = a.dm.r, tid = threadIdx.x;
  {
    constexpr int NG = kEncThreads / D, R = kTE / NG;
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
    for (int i = 0; i < R; ++i) vh[(tg + NG * i) * D + j] = acc[i];   // K~_pre for now
  }
  __syncthreads();
  {
    constexpr int NG = kEncThreads / FH, R = kTE / NG;
    const int f = tid % FH, tg = tid / FH;
    const T* wrow = (const T*)a.w1 + ((size_t)h * FH + f) * D;
    float acc[R];
#pragma unroll
    for (int i = 0; i < R; ++i) acc[i] = 0.f;
    for (int j = 0; j < D; ++j) {
      const float w = ldf(wrow, j);
#pragma unroll
      for (int i = 0; i < R; ++i) acc[i] = fmaf(w, vh[(tg + NG * i) * D + j], acc[i]);
    }
    const float bias = ldf((const T*)a.b1, (size_t)h * FH + f);
#pragma unroll
    for (int i = 0; i < R; ++i) hid[(tg + NG * i) * FH + f] = act_f(acc[i] + bias, a.dm.act);
  }
  __syncthreads();
  {
    constexpr int NG = kEncThreads / D, R = kTE / NG;
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
    for (int i = 0; i < R; ++i) vh[(tg + NG * i) * D + j] = acc[i] + bias;
  }
  __syncthreads();
}

// E1 + E2 + E4 for kTE tokens of one batch element.
template <typename T, int D, int FH>
__global__ void __launch_bounds__(kEncThreads) project_error_kernel(const EncodeArgs a) {
  const Dims& dm = a.dm;
  const int b = blockIdx.y, t0 = blockIdx.x * kTE, tid = threadIdx.x;
  const int H = dm.H, r = dm.r, Dt = H * D;
  extern __shared__ float sm[];
  float* kp = sm;                 // [kTE][Dt]
  float* cs = kp + kTE * Dt;      // [kTE][r]
  float* vh = cs + kTE * r;       // [kTE][D]
  float* hid = vh + kTE * D;      // [kTE][FH]
  const T* kc = (const T*)a.k_cache;

  // E1: inverse rotation, pairs (i, i + D/2) of every head
  for (int o = tid; o < kTE * H * (D / 2); o += blockDim.x) {
    const int i = o % (D / 2);
    const int h = (o / (D / 2)) % H;
    const int t = o / ((D / 2) * H);
    const size_t base = (((size_t)b * dm.T + t0 + t) * H + h) * D;
    const float x = ldf(kc, base + i), y = ldf(kc, base + i + D / 2);
    const float2 c2 = rope_cs32(a.rope, i, token_position(dm, a.chunk_pos, b, t0 + t, a.status));
    kp[t * Dt + h * D + i] = x * c2.x + y * c2.y;
    kp[t * Dt + h * D + i + D / 2] = y * c2.x - x * c2.y;
  }
  __syncthreads();
  // E2: projection onto the basis
  if (tid < r) {
    float acc[kTE];
#pragma unroll
    for (int t = 0; t < kTE; ++t) acc[t] = 0.f;
    const T* bcol = (const T*)a.basis + tid;
    for (int i = 0; i < Dt; ++i) {
      const float bv = ldf(bcol, (size_t)i * r);
#pragma unroll
      for (int t = 0; t < kTE; ++t) acc[t] = fmaf(bv, kp[t * Dt + i], acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kTE; ++t) {
      cs[t * r + tid] = acc[t];
      ((T*)a.coef)[((size_t)b * dm.T + t0 + t) * r + tid] = from_f<T>(acc[t]);
    }
  }
  __syncthreads();
  // E4: per head, predictor on the rebuilt key and squared error against V
  const T* vin = (const T*)a.v;
  const int warp = tid >> 5, lane = tid & 31;
  for (int h = 0; h < H; ++h) {
    predict_tile<T, D, FH>(a, h, cs, vh, hid);
    for (int o = tid; o < kTE * D; o += blockDim.x) {
      const int t = o / D, j = o - t * D;
      const float dv = ldf(vin, (((size_t)b * dm.T + t0 + t) * H + h) * D + j) - vh[o];
      vh[o] = dv * dv;
    }
    __syncthreads();
    for (int t = warp; t < kTE; t += kEncThreads / 32) {
      float s = 0.f;
      for (int j = lane; j < D; j += 32) s += vh[t * D + j];
      s = warp_sum(s);
      if (lane == 0) a.err[((size_t)b * H + h) * dm.T + t0 + t] = s;
    }
    __syncthreads();
  }
}

// E5a: per (b, h) threshold and classification. flags: 1 = in, 2 = fp64 candidate.
__global__ void __launch_bounds__(kSelEncThreads) residual_threshold_kernel(const EncodeArgs a) {
  const Dims& dm = a.dm;
  const int p = blockIdx.x, T = dm.T, tid = threadIdx.x;
  const float* e = a.err + (size_t)p * T;
  uint8_t* flags = a.flags + (size_t)p * T;
  int* cidx = a.cand_idx + (size_t)p * T;
  __shared__ unsigned hist[256];
  __shared__ unsigned bc[4];
  __shared__ float fscr[33];
  __shared__ int iscr[33];
  __shared__ int cnt;
  if (dm.n_res == 0 || dm.n_res >= T) {
    const uint8_t f = dm.n_res == 0 ? 0 : 1;
    for (int i = tid; i < T; i += blockDim.x) flags[i] = f;
    if (tid == 0) { a.cand_count[p] = 0; a.in_count[p] = dm.n_res == 0 ? 0 : T; }
    return;
  }
  float mx = 0.f;
  for (int i = tid; i < T; i += blockDim.x) mx = fmaxf(mx, fabsf(e[i]));
  mx = group_max(whole_block(), mx, fscr);
  const uint32_t tk = group_kth_largest(whole_block(), T, dm.n_res,
                                        [&](int i) { return f2key(e[i]); }, hist, bc);
  const double tau = (double)key2f(tk);
  const double delta = 2e-3 * fabs(tau) + 1e-6 * (double)mx + 1e-30;
  const double hi = tau + delta, lo = tau - delta;
  if (tid == 0) cnt = 0;
  __syncthreads();
  int n_in = 0;
  for (int i = tid; i < T; i += blockDim.x) {
    const double x = (double)e[i];
    uint8_t f = 0;
    if (x > hi) {
      f = 1;
      ++n_in;
    } else if (x >= lo) {
      f = 2;
      cidx[atomicAdd(&cnt, 1)] = i;
    }
    flags[i] = f;
  }
  int total;
  (void)group_exclusive_scan(whole_block(), n_in, iscr, &total);
  if (tid == 0) { a.in_count[p] = total; a.cand_count[p] = cnt; }
}

// E5b: fp64 error of every candidate: the whole chain recomputed in fp64 from the
// stored inputs (inputs widen exactly; fp64 RoPE tables; fp64 exp / erf), for a batch of
// kNB candidates of one (b, h) per pass, so that every basis and weight element staged in
// shared memory serves all kNB of them:
//   c = B^T RoPE^-1(K)     (over the D = H d columns, one head's block at a time)
//   K~ = B_h c;  hid = act(W1_h K~ + b1);  V_hat = W2_h hid + b2;  e = |V - V_hat|^2
// Each product is a small GEMM with a 4 (candidates) x m (columns) register tile per
// thread; the weights are staged transposed where that keeps the lanes' reads in
// consecutive banks.
constexpr int kNB = 32;   // candidates per pass

// Bytes of the re-score's staging region B: the largest operand staged there, a head's
// basis block [D][r] (or its transpose), W1_h^T [D][FH] or W2_h^T [FH][D], in T.
template <typename T>
__host__ __device__ constexpr size_t rescore_stage_bytes(int D, int r, int FH) {
  return (size_t)D * (size_t)(r > FH ? r : FH) * sizeof(T);   // a multiple of 16 bytes
}

template <typename T>
__device__ __forceinline__ double ld64(const T* p, size_t i) { return (double)to_f(p[i]); }


// MC: 32-column blocks of c per lane, ceil(r / 32) when it is known at compile time (the
// projection loop then runs no predicated-off blocks), 8 for any r <= 256 otherwise.
template <typename T, int D, int FH, int MC>
__global__ void __launch_bounds__(kEncThreads) residual_rescore_kernel(const EncodeArgs a) {
  const Dims& dm = a.dm;
  const int p = blockIdx.y, b = p / dm.H, h = p % dm.H, tid = threadIdx.x;
  const int H = dm.H, r = dm.r;
  const int n = a.cand_count[p];
  extern __shared__ double smd[];
  // region A: [kNB][D] fp64 (pre-RoPE keys of one head, later K~)
  // region B: staged operands (basis block, transposed basis_h, W1^T, W2^T), sized for
  //           the largest of them
  // region C: [kNB][max(r, FH)] fp64 (c, later hid)
  double* sA = smd;
  T* sB = reinterpret_cast<T*>(smd + kNB * D);
  double* sC = smd + kNB * D + rescore_stage_bytes<T>(D, r, FH) / 8;
  __shared__ int s_tok[kNB];
  __shared__ double s_e[kNB];
  const int cg = tid >> 5, lane = tid & 31;     // candidate group (4 each), column lane
  const T* kc = (const T*)a.k_cache;
  const T* basis = (const T*)a.basis;
  for (int j0 = blockIdx.x * kNB; j0 < n; j0 += gridDim.x * kNB) {
    const int nb = min(kNB, n - j0);
    if (tid < kNB) s_tok[tid] = tid < nb ? a.cand_idx[(size_t)p * dm.T + j0 + tid] : -1;
    __syncthreads();
    // ---- c[cand][kk] = sum over heads hh, dims i of kpre[cand][hh d + i] basis[hh d + i][kk]
    constexpr int kMaxC = MC;   // columns per lane
    double acc[4][kMaxC];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int m = 0; m < kMaxC; ++m) acc[x][m] = 0.0;
    // this thread's RoPE^-1 work in every head: candidate kc_c, rotary pairs kc_i0 ..
    // kc_i0 + 7 (the same positions in every head, so their rotations are read once)
    constexpr int kBlk = D / 16;   // blocks of 8 rotary pairs per candidate
    const bool kc_act = tid < kNB * kBlk;
    const int kc_c = kc_act ? tid / kBlk : 0, kc_i0 = (tid % kBlk) * 8;
    const int kc_t = kc_act ? s_tok[kc_c] : -1;
    double cs8[8], sn8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { cs8[e] = 1.0; sn8[e] = 0.0; }
    if (kc_t >= 0) {
      const int pos = token_position(dm, a.chunk_pos, b, kc_t, a.status);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const double2 c2 = rope_cs64(a.rope, kc_i0 + e, pos);
        cs8[e] = c2.x;
        sn8[e] = c2.y;
      }
    }
    // A head's operands: this thread's key slices and its share of the basis block
    // [D][r] (contiguous, 16-byte units). When the share fits in registers, the next
    // head's are loaded while this head's products run.
    constexpr int kBV = (int)(((size_t)D * 32 * MC * sizeof(T) / 16 + kEncThreads - 1) / kEncThreads);
    constexpr bool kPrefetch = kBV <= 16;
    const int n16 = (int)((size_t)D * r * sizeof(T) / 16);
    T xr[8], yr[8];
    uint4 bv16[kPrefetch ? kBV : 1];
    auto load_keys = [&](int hh) {
      if (kc_act && kc_t >= 0) {
        const T* krow = kc + (((size_t)b * dm.T + kc_t) * H + hh) * D;
        ld8_raw(krow + kc_i0, xr);
        ld8_raw(krow + kc_i0 + D / 2, yr);
      }
    };
    auto load_basis = [&](int hh) {
      const uint4* src = reinterpret_cast<const uint4*>(basis + (size_t)hh * D * r);
#pragma unroll
      for (int q = 0; q < (kPrefetch ? kBV : 1); ++q) {
        const int o = tid + q * kEncThreads;
        if (o < n16) bv16[q] = __ldg(src + o);
      }
    };
    auto store_operands = [&](int hh) {
      if (kc_act) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const double x = kc_t >= 0 ? (double)to_f(xr[e]) : 0.0;
          const double y = kc_t >= 0 ? (double)to_f(yr[e]) : 0.0;
          sA[kc_c * D + kc_i0 + e] = x * cs8[e] + y * sn8[e];
          sA[kc_c * D + kc_i0 + e + D / 2] = y * cs8[e] - x * sn8[e];
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(sB);
      if constexpr (kPrefetch) {
#pragma unroll
        for (int q = 0; q < kBV; ++q) {
          const int o = tid + q * kEncThreads;
          if (o < n16) dst[o] = bv16[q];
        }
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(basis + (size_t)hh * D * r);
#pragma unroll 4
        for (int o = tid; o < n16; o += kEncThreads) dst[o] = __ldg(src + o);
      }
    };
    load_keys(0);
    if constexpr (kPrefetch) load_basis(0);
    for (int hh = 0; hh < H; ++hh) {
      __syncthreads();   // the previous head's operands are consumed
      if (!kPrefetch) load_keys(hh);
      store_operands(hh);
      __syncthreads();
      if (kPrefetch && hh + 1 < H) {   // in flight under this head's products
        load_keys(hh + 1);
        load_basis(hh + 1);
      }
      for (int i = 0; i < D; ++i) {
        double kv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) kv[x] = sA[(4 * cg + x) * D + i];
#pragma unroll
        for (int m = 0; m < kMaxC; ++m) {
          const int kk = lane + 32 * m;
          if (kk < r) {
            const double bv = (double)to_f(sB[i * r + kk]);
#pragma unroll
            for (int x = 0; x < 4; ++x) acc[x][m] = fma(kv[x], bv, acc[x][m]);
          }
        }
      }
    }
    __syncthreads();
    // c to region C; the head's basis block transposed into region B: sB[kk][j] = B_h[j][kk]
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int m = 0; m < kMaxC; ++m) {
        const int kk = lane + 32 * m;
        if (kk < r) sC[(4 * cg + x) * r + kk] = acc[x][m];
      }
#pragma unroll 2
    for (int o = tid; o < D * r / 8; o += blockDim.x) {   // 8 consecutive kk of row j
      const int j = o / (r / 8), kk0 = (o % (r / 8)) * 8;
      T v[8];
      ld8_raw(basis + ((size_t)h * D + j) * r + kk0, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) sB[(kk0 + e) * D + j] = v[e];
    }
    __syncthreads();
    // ---- K~[cand][j] = sum_kk c[cand][kk] B_h[j][kk]  (into region A)
    {
      constexpr int M = D / 32;
      double kt[4][M];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int m = 0; m < M; ++m) kt[x][m] = 0.0;
      for (int kk = 0; kk < r; ++kk) {
        double cv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) cv[x] = sC[(4 * cg + x) * r + kk];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const double bv = (double)to_f(sB[kk * D + lane + 32 * m]);
#pragma unroll
          for (int x = 0; x < 4; ++x) kt[x][m] = fma(cv[x], bv, kt[x][m]);
        }
      }
      __syncthreads();   // region B (basis_h) and C (c) consumed; A is overwritten now
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int m = 0; m < M; ++m) sA[(4 * cg + x) * D + lane + 32 * m] = kt[x][m];
    }
    // W1_h transposed into region B: sB[j][f] = W1[h][f][j]
#pragma unroll 2
    for (int o = tid; o < FH * D / 8; o += blockDim.x) {   // 8 consecutive j of row f
      const int f = o / (D / 8), j0 = (o % (D / 8)) * 8;
      T v[8];
      ld8_raw((const T*)a.w1 + ((size_t)h * FH + f) * D + j0, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) sB[(j0 + e) * FH + f] = v[e];
    }
    __syncthreads();
    // ---- hid[cand][f] = act(sum_j K~[cand][j] W1[f][j] + b1[f])  (into region C)
    {
      constexpr int M = FH / 32;
      double hv[4][M];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int m = 0; m < M; ++m) hv[x][m] = ld64((const T*)a.b1, (size_t)h * FH + lane + 32 * m);
      for (int j = 0; j < D; ++j) {
        double kv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) kv[x] = sA[(4 * cg + x) * D + j];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const double wv = (double)to_f(sB[j * FH + lane + 32 * m]);
#pragma unroll
          for (int x = 0; x < 4; ++x) hv[x][m] = fma(kv[x], wv, hv[x][m]);
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int m = 0; m < M; ++m) sC[(4 * cg + x) * FH + lane + 32 * m] = act_d(hv[x][m], dm.act);
    }
    __syncthreads();   // region B (W1) consumed
    // W2_h transposed into region B: sB[f][j] = W2[h][j][f]
#pragma unroll 2
    for (int o = tid; o < D * FH / 8; o += blockDim.x) {   // 8 consecutive f of row j
      const int j = o / (FH / 8), f0 = (o % (FH / 8)) * 8;
      T v[8];
      ld8_raw((const T*)a.w2 + ((size_t)h * D + j) * FH + f0, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) sB[(f0 + e) * D + j] = v[e];
    }
    __syncthreads();
    // ---- V_hat[cand][j] = sum_f hid[cand][f] W2[j][f] + b2[j];  e = sum_j (V - V_hat)^2
    {
      constexpr int M = D / 32;
      double ov[4][M];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int m = 0; m < M; ++m) ov[x][m] = ld64((const T*)a.b2, (size_t)h * D + lane + 32 * m);
      for (int f = 0; f < FH; ++f) {
        double hvv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) hvv[x] = sC[(4 * cg + x) * FH + f];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const double wv = (double)to_f(sB[f * D + lane + 32 * m]);
#pragma unroll
          for (int x = 0; x < 4; ++x) ov[x][m] = fma(hvv[x], wv, ov[x][m]);
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int c = 4 * cg + x;
        const int t = s_tok[c];
        double sq = 0.0;
        if (t >= 0) {
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const double dv = ld64((const T*)a.v, (((size_t)b * dm.T + t) * H + h) * D + lane + 32 * m) - ov[x][m];
            sq = fma(dv, dv, sq);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_e[c] = sq;
      }
    }
    __syncthreads();
    if (tid < nb) a.cand_e64[(size_t)p * dm.T + j0 + tid] = s_e[tid];
    __syncthreads();
  }
}

// E5c: exact ranking of the candidates, ascending compaction, chunk CSR.
__global__ void __launch_bounds__(kSelEncThreads) residual_finalize_kernel(const EncodeArgs a) {
  const Dims& dm = a.dm;
  const int p = blockIdx.x, T = dm.T, tid = threadIdx.x;
  uint8_t* flags = a.flags + (size_t)p * T;
  const int* cidx = a.cand_idx + (size_t)p * T;
  const double* ce = a.cand_e64 + (size_t)p * T;
  int32_t* ridx = a.res_idx + (size_t)p * dm.n_res;
  int32_t* ptr = a.chunk_ptr + (size_t)p * (dm.Nc + 1);
  __shared__ int iscr[33];
  const int n_w = a.cand_count[p];
  const int need = dm.n_res - a.in_count[p];
  for (int j = tid; j < n_w; j += blockDim.x) {
    const double sj = ce[j];
    const int ij = cidx[j];
    int rank = 0;
    for (int m = 0; m < n_w; ++m) {
      const double sm = ce[m];
      rank += (sm > sj) || (sm == sj && cidx[m] < ij);
    }
    flags[ij] = rank < need ? 1 : 0;
  }
  __syncthreads();
  int base = 0;
  for (int c0 = 0; c0 < T; c0 += blockDim.x) {
    const int i = c0 + tid;
    const int f = (i < T && flags[i] == 1) ? 1 : 0;
    int total;
    const int ex = group_exclusive_scan(whole_block(), f, iscr, &total);
    if (f && base + ex < dm.n_res) ridx[base + ex] = i;
    base += total;
  }
  __syncthreads();
  // ptr[c] = number of residual tokens below c*C (binary search in the ascending list)
  for (int c = tid; c <= dm.Nc; c += blockDim.x) {
    const int key = c * dm.C;
    int lo = 0, hi = dm.n_res;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ridx[mid] < key) lo = mid + 1; else hi = mid;
    }
    ptr[c] = lo;
  }
}

// E6: residual rows against the STORED coefficients.
template <typename T, int D, int FH>
__global__ void __launch_bounds__(kEncThreads) residual_rows_kernel(const EncodeArgs a) {
  const Dims& dm = a.dm;
  const int p = blockIdx.y, b = p / dm.H, h = p % dm.H, tid = threadIdx.x;
  const int r = dm.r, s0 = blockIdx.x * kTE;
  extern __shared__ float sm[];
  float* cs = sm;                 // [kTE][r]
  float* vh = cs + kTE * r;       // [kTE][D]
  float* hid = vh + kTE * D;      // [kTE][FH]
  __shared__ int s_tok[kTE];
  const int32_t* ridx = a.res_idx + (size_t)p * dm.n_res;
  if (tid < kTE) s_tok[tid] = (s0 + tid < dm.n_res) ? ridx[s0 + tid] : -1;
  __syncthreads();
  for (int o = tid; o < kTE * r; o += blockDim.x) {
    const int t = o / r, kk = o - t * r;
    const int tok = s_tok[t];
    cs[o] = tok >= 0 ? ldf((const T*)a.coef, ((size_t)b * dm.T + tok) * r + kk) : 0.f;
  }
  __syncthreads();
  predict_tile<T, D, FH>(a, h, cs, vh, hid);
  for (int o = tid; o < kTE * D; o += blockDim.x) {
    const int t = o / D, j = o - t * D;
    const int tok = s_tok[t];
    if (tok < 0) continue;
    const float v = ldf((const T*)a.v, (((size_t)b * dm.T + tok) * dm.H + h) * D + j);
    ((T*)a.res_val)[((size_t)p * dm.n_res + s0 + t) * D + j] = from_f<T>(v - vh[o]);
  }
}

template <typename T, int D, int FH>
cudaError_t launch_encode_typed(const EncodeArgs& a, cudaStream_t s) {
  const Dims& dm = a.dm;
  cudaError_t e;
  {
    const size_t n8 = (size_t)dm.B * dm.H * dm.Nc * dm.d / 8;
    const int blocks = (int)((n8 + 255) / 256 < 65535 * 8 ? (n8 + 255) / 256 : 65535 * 8);
    landmark_kernel<T><<<blocks, 256, 0, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const bool tc = a.c_ws != nullptr && encode_tc_supported(dm);
  if (tc) {   // E1 + E2 and E4 on the tensor cores
    if ((e = launch_encode_project_tc(a, a.basis_t, a.c_ws, a.num_sms, s)) != cudaSuccess) return e;
    if ((e = launch_encode_predict_tc(a, a.c_ws, false, a.num_sms, s)) != cudaSuccess) return e;
  } else {
    const size_t smem = sizeof(float) * ((size_t)kTE * dm.H * D + (size_t)kTE * dm.r +
                                         kTE * D + kTE * FH);
    auto kern = project_error_kernel<T, D, FH>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess) return e;
    kern<<<dim3(dm.T / kTE, dm.B), kEncThreads, smem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  residual_threshold_kernel<<<dm.B * dm.H, kSelEncThreads, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    const int wc = dm.r > FH ? dm.r : FH;
    const size_t smem = sizeof(double) * ((size_t)kNB * D + (size_t)kNB * wc) +
                        rescore_stage_bytes<T>(D, dm.r, FH);   // <= 224 KB (d <= 128, r, F <= 256)
    auto kern = dm.r == 160   ? residual_rescore_kernel<T, D, FH, 5>
                : dm.r == 128 ? residual_rescore_kernel<T, D, FH, 4>
                              : residual_rescore_kernel<T, D, FH, 8>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess) return e;
    kern<<<dim3(kRescoreCtas, dm.B * dm.H), kEncThreads, smem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  residual_finalize_kernel<<<dm.B * dm.H, kSelEncThreads, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (dm.n_res > 0 && tc) {   // E6 on the tensor cores
    if ((e = launch_encode_predict_tc(a, a.c_ws, true, a.num_sms, s)) != cudaSuccess) return e;
  } else if (dm.n_res > 0) {
    const size_t smem = sizeof(float) * ((size_t)kTE * dm.r + kTE * D + kTE * FH);
    auto kern = residual_rows_kernel<T, D, FH>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess) return e;
    kern<<<dim3((dm.n_res + kTE - 1) / kTE, dm.B * dm.H), kEncThreads, smem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

// landmark_norm[p] = max over chunks of |L_pc|_2 (exact squares, fp64 sums), rounded up
// to fp32 with a margin for the fp64 rounding.
template <typename T>
__global__ void __launch_bounds__(256) landmark_norm_kernel(const Dims dm, const T* landmark,
                                                            float* norm) {
  // CTA (x, p): landmark rows [kNormRows x, kNormRows (x + 1)) of (b, h) pair p; d / 8
  // lanes per row (8 elements each), squares summed in fp64. Each CTA raises norm[p] to its own
  // rounded-up bound with an integer max on the (non-negative) fp32 bits, so the result
  // is the bound of the largest row: rounding up and the square root are monotonic.
  const int p = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* Lp = landmark + (size_t)p * dm.Nc * dm.d;
  const int c_end = min(dm.Nc, (int)(blockIdx.x + 1) * kNormRows);
  const int per_row = dm.d / 8;   // lanes per row (16 at d = 128, 8 at d = 64)
  const int rows_per_warp = 32 / per_row;
  double best = 0.0;
  for (int c0 = blockIdx.x * kNormRows + warp * rows_per_warp; c0 < c_end;
       c0 += (blockDim.x >> 5) * rows_per_warp) {
    const int c = c0 + lane / per_row;
    double ss = 0.0;
    if (c < c_end) {
      T v[8];
      ld8_raw(Lp + (size_t)c * dm.d + 8 * (lane % per_row), v);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const double x = (double)to_f(v[e]);
        ss = fma(x, x, ss);
      }
    }
    for (int o = per_row / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    best = fmax(best, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = fmax(best, __shfl_xor_sync(0xffffffffu, best, o));
  __shared__ double wmax[8];
  if (lane == 0) wmax[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) best = fmax(best, wmax[w]);
    const float bound = __double2float_ru(sqrt(best) * (1.0 + 1e-12));
    atomicMax(reinterpret_cast<unsigned int*>(norm + p), __float_as_uint(bound));
  }
}

cudaError_t launch_landmark_norms(const Dims& dm, const void* landmark, float* norm,
                                  cudaStream_t s) {
  const int pairs = dm.B * dm.H;
  cudaError_t e = cudaMemsetAsync(norm, 0, (size_t)pairs * sizeof(float), s);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((dm.Nc + kNormRows - 1) / kNormRows), (unsigned)pairs);
  if (dm.dtype == LOWRAM_DTYPE_BF16)
    landmark_norm_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(dm, (const __nv_bfloat16*)landmark, norm);
  else
    landmark_norm_kernel<float><<<grid, 256, 0, s>>>(dm, (const float*)landmark, norm);
  return cudaGetLastError();
}

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s) {
  const bool bf = a.dm.dtype == LOWRAM_DTYPE_BF16;
  const int D = a.dm.d, FH = a.dm.F;
#define LR_CASE(DD, FF)                                                    \
  if (D == DD && FH == FF)                                                 \
    return bf ? launch_encode_typed<__nv_bfloat16, DD, FF>(a, s)           \
              : launch_encode_typed<float, DD, FF>(a, s);
  LR_CASE(64, 128) LR_CASE(64, 256) LR_CASE(128, 128) LR_CASE(128, 256)
#undef LR_CASE
  return cudaErrorInvalidValue;
}

}  // namespace lowram
