// Eviction before compression (LowRAM-E / LowRAM-EQ: the method composes with eviction,
// agihunt summary, composition paragraph; eviction shortens the sequence).
//
// For every batch element, the chunks of the P-position prefix are ranked by their
// all-head landmark norm, sum_h |L_c,h|^2, with the landmarks computed exactly as the
// encode stores them (fp32 chunk mean of the keys, rounded to the cache dtype) and the
// squares summed in fp64. The T / C largest are kept (ties to the lower chunk), in
// ascending order, and their keys and values are copied out; chunk_pos records each kept
// chunk's original index, so RoPE is later inverted and re-applied at the original
// positions.
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace lowram {
namespace {

constexpr int kNormThreads = 256;
constexpr int kRankThreads = 256;
constexpr int kRankTile = 2048;

// norm[b * Pc + c] = sum over heads and dims of landmark^2 (one warp per chunk)
template <typename T>
__global__ void __launch_bounds__(kNormThreads) evict_norm_kernel(const Dims dm, const T* k,
                                                                  double* norm) {
  const int Pc = dm.P / dm.C;
  const int w = blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= dm.B * Pc) return;
  const int b = w / Pc, c = w % Pc;
  const int HD = dm.H * dm.d;
  double ss = 0.0;
  for (int idx = lane; idx < HD; idx += 32) {
    float acc = 0.f;
    for (int i = 0; i < dm.C; ++i)
      acc += ldf(k, ((size_t)b * dm.P + (size_t)c * dm.C + i) * HD + idx);
    const double lm = (double)to_f(from_f<T>(acc / (float)dm.C));
    ss = fma(lm, lm, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) norm[w] = ss;
}

// keep[b * Pc + c] = 1 when fewer than Nc chunks of b rank above c (larger norm, or equal
// norm and lower index)
__global__ void __launch_bounds__(kRankThreads) evict_rank_kernel(const Dims dm, const double* norm,
                                                                  uint8_t* keep) {
  const int Pc = dm.P / dm.C, b = blockIdx.y;
  const int c = blockIdx.x * kRankThreads + threadIdx.x;
  const double* nb = norm + (size_t)b * Pc;
  const double mine = c < Pc ? nb[c] : 0.0;
  __shared__ double tile[kRankTile];
  int rank = 0;
  for (int t0 = 0; t0 < Pc; t0 += kRankTile) {
    const int n = min(kRankTile, Pc - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kRankThreads) tile[i] = nb[t0 + i];
    __syncthreads();
    if (c < Pc) {
      for (int i = 0; i < n; ++i) {
        const double o = tile[i];
        rank += (o > mine) || (o == mine && t0 + i < c);
      }
    }
  }
  if (c < Pc) keep[(size_t)b * Pc + c] = rank < dm.Nc ? 1 : 0;
}

// chunk_pos[b][slot] = the slot-th kept chunk of b (one CTA per batch element)
__global__ void __launch_bounds__(1024) evict_compact_kernel(const Dims dm, const uint8_t* keep,
                                                             int32_t* chunk_pos) {
  const int Pc = dm.P / dm.C, b = blockIdx.x;
  __shared__ int iscr[33];
  int base = 0;
  for (int c0 = 0; c0 < Pc; c0 += blockDim.x) {
    const int c = c0 + threadIdx.x;
    const int f = (c < Pc && keep[(size_t)b * Pc + c]) ? 1 : 0;
    int total;
    const int ex = group_exclusive_scan(whole_block(), f, iscr, &total);
    if (f && base + ex < dm.Nc) chunk_pos[(size_t)b * dm.Nc + base + ex] = c;
    base += total;
  }
}

// row (b, t) of the kept cache <- row (b, chunk_pos*C + t % C) of the full prefix
__global__ void __launch_bounds__(128) evict_gather_kernel(const Dims dm, const uint4* k,
                                                           const uint4* v, uint4* kk, uint4* vv,
                                                           const int32_t* chunk_pos,
                                                           int row_vec) {
  const size_t row = blockIdx.x;   // b * T + t
  const int b = (int)(row / dm.T), t = (int)(row % dm.T);
  const int src = chunk_pos[(size_t)b * dm.Nc + t / dm.C] * dm.C + t % dm.C;
  const size_t so = ((size_t)b * dm.P + src) * row_vec, dst = row * row_vec;
  for (int i = threadIdx.x; i < row_vec; i += blockDim.x) {
    kk[dst + i] = k[so + i];
    vv[dst + i] = v[so + i];
  }
}

}  // namespace

size_t evict_workspace_bytes(const Dims& dm) {
  const size_t n = (size_t)dm.B * (dm.P / dm.C);
  return (n * sizeof(double) + 255) / 256 * 256 + n;
}

cudaError_t launch_evict(const Dims& dm, const void* k_full, const void* v_full, void* k_kept,
                         void* v_kept, int32_t* chunk_pos, void* ws, cudaStream_t s) {
  const int Pc = dm.P / dm.C;
  const size_t n = (size_t)dm.B * Pc;
  double* norm = static_cast<double*>(ws);
  uint8_t* keep = static_cast<uint8_t*>(ws) + (n * sizeof(double) + 255) / 256 * 256;
  const int nb = (int)((n + kNormThreads / 32 - 1) / (kNormThreads / 32));
  if (dm.dtype == LOWRAM_DTYPE_BF16)
    evict_norm_kernel<__nv_bfloat16><<<nb, kNormThreads, 0, s>>>(dm, (const __nv_bfloat16*)k_full, norm);
  else
    evict_norm_kernel<float><<<nb, kNormThreads, 0, s>>>(dm, (const float*)k_full, norm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  evict_rank_kernel<<<dim3((Pc + kRankThreads - 1) / kRankThreads, dm.B), kRankThreads, 0, s>>>(
      dm, norm, keep);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  evict_compact_kernel<<<dm.B, 1024, 0, s>>>(dm, keep, chunk_pos);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int es = dm.dtype == LOWRAM_DTYPE_BF16 ? 2 : 4;
  const int row_vec = dm.H * dm.d * es / 16;
  evict_gather_kernel<<<(unsigned)((size_t)dm.B * dm.T), 128, 0, s>>>(
      dm, (const uint4*)k_full, (const uint4*)v_full, (uint4*)k_kept, (uint4*)v_kept, chunk_pos,
      row_vec);
  return cudaGetLastError();
}

}  // namespace lowram
