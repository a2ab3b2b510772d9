// Kernel (a): landmark scoring and top-k chunk selection for one decode step.
//
// Method: the prefix is cut into chunks whose mean key is a landmark; each decode step
// scores the landmarks with the current query and rebuilds only the top-k chunks
// (LowRAM summary on agihunt.info, paragraph on the key side; cctest "How the method
// works", Selective reconstruction). With GQA a chunk's score is the max over the
// group's query heads of q . L_c; ties go to the lower chunk index.
//
// Structure (HBM-bound: every landmark byte is read once; ~4 FLOP per byte):
//  * grid (n_slices, B*H_kv); a CTA scores one slice of one (batch, KV head).
//    Each warp streams groups of U = 32/G landmarks; lane l holds dims
//    [l*E, l*E+E) of the G queries in registers (E = d/32) and of each landmark, so the
//    loads are coalesced rows. The U*G partial dot products of a group are summed across
//    lanes by a reduce-scatter (31 shuffles per 32 values) that leaves lane l with value
//    l; a max over G lanes gives the chunk score, written as fp32.
//  * The last CTA of a (batch, KV head) to finish (atomic counter, no spinning) selects:
//    radix select of the k-th largest fp32 score tau; chunks with score > tau + delta are
//    in, chunks within delta of tau are re-scored in fp64 (exact products, fp64 sums)
//    and ranked by (fp64 score desc, index asc). delta = 1e-3|tau| + 1e-6 max|s| is far
//    above the fp32 accumulation error, so the result equals the fp64 selection.
//    The selection is written in ascending chunk order.
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace lowram {
namespace {

constexpr int kSelThreads = 256;

// One reduce-scatter step: 2N values per lane -> N, exchanging the half this lane
// does not keep with the partner lane^off.
template <int N>
__device__ __forceinline__ void rs_step(float* v, bool upper, int off) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float send = upper ? v[i] : v[i + N];
    const float keep = upper ? v[i + N] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
  }
}

template <typename T, int D, int G>
__device__ double score64(const T* lrow, const T* qb) {
  double best = -INFINITY;
  for (int g = 0; g < G; ++g) {
    double acc = 0.0;
    for (int j = 0; j < D; ++j) acc += ldd(qb, g * D + j) * ldd(lrow, j);
    best = fmax(best, acc);
  }
  return best;
}

template <typename T, int D, int G>
__device__ void select_pair(const SelectArgs& a, int p) {
  const Dims& dm = a.dm;
  const int Nc = dm.Nc, k = dm.k;
  int32_t* sel = a.sel + (size_t)p * k;
  const int tid = threadIdx.x;
  if (k >= Nc) {
    for (int i = tid; i < Nc; i += blockDim.x) sel[i] = i;
    return;
  }
  __shared__ unsigned hist[256];
  __shared__ unsigned bc[4];
  __shared__ float fscr[33];
  __shared__ int iscr[33];
  __shared__ int cnt[2];
  const float* s = a.scores + (size_t)p * Nc;
  uint8_t* flags = a.flags + (size_t)p * Nc;
  int* cidx = a.cand_idx + (size_t)p * Nc;
  double* cs64 = a.cand_s64 + (size_t)p * Nc;

  float mx = 0.f;
  for (int i = tid; i < Nc; i += blockDim.x) mx = fmaxf(mx, fabsf(__ldcg(s + i)));
  mx = block_max(mx, fscr);

  const uint32_t tk = block_kth_largest(
      Nc, k, [&](int i) { return f2key(__ldcg(s + i)); }, hist, bc);
  const double tau = (double)key2f(tk);
  const double delta = 1e-3 * fabs(tau) + 1e-6 * (double)mx + 1e-30;
  const double hi = tau + delta, lo = tau - delta;

  if (tid == 0) { cnt[0] = 0; cnt[1] = 0; }
  __syncthreads();
  const int b = p / dm.H, h = p % dm.H;
  const T* qb = (const T*)a.q + ((size_t)b * dm.Hq + (size_t)h * G) * D;
  const T* L = (const T*)a.landmark + (size_t)p * Nc * D;
  int n_in = 0;
  for (int i = tid; i < Nc; i += blockDim.x) {
    const double x = (double)__ldcg(s + i);
    uint8_t f = 0;
    if (x > hi) {
      f = 1;
      ++n_in;
    } else if (x >= lo) {
      f = 2;
      const int slot = atomicAdd(&cnt[1], 1);
      cidx[slot] = i;
      cs64[slot] = score64<T, D, G>(L + (size_t)i * D, qb);
    }
    flags[i] = f;
  }
  int n_in_total;
  (void)block_exclusive_scan(n_in, iscr, &n_in_total);
  const int n_w = cnt[1];
  const int need = k - n_in_total;
  // rank the window candidates by (fp64 score desc, index asc); keep the first `need`
  for (int j = tid; j < n_w; j += blockDim.x) {
    const double sj = cs64[j];
    const int ij = cidx[j];
    int rank = 0;
    for (int m = 0; m < n_w; ++m) {
      const double sm = cs64[m];
      rank += (sm > sj) || (sm == sj && cidx[m] < ij);
    }
    flags[ij] = rank < need ? 1 : 0;
  }
  __syncthreads();
  int base = 0;
  for (int c0 = 0; c0 < Nc; c0 += blockDim.x) {
    const int i = c0 + tid;
    const int f = (i < Nc && flags[i] == 1) ? 1 : 0;
    int total;
    const int ex = block_exclusive_scan(f, iscr, &total);
    if (f && base + ex < k) sel[base + ex] = i;
    base += total;
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kSelThreads, 3) score_select_kernel(const SelectArgs a) {
  constexpr int E = D / 32;
  constexpr int U = 32 / G;
  const Dims& dm = a.dm;
  const int p = blockIdx.y;
  const int b = p / dm.H, h = p % dm.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Nc = dm.Nc;
  const T* L = (const T*)a.landmark + (size_t)p * Nc * D + lane * E;

  float qr[G][E];
  {
    const T* qp = (const T*)a.q + ((size_t)b * dm.Hq + (size_t)h * G) * D + lane * E;
#pragma unroll
    for (int g = 0; g < G; ++g) VecLoad<T, E>::load(qp + g * D, qr[g]);
  }
  const int c_begin = blockIdx.x * a.slice_len;
  const int c_end = min(Nc, c_begin + a.slice_len);
  float* out = a.scores + (size_t)p * Nc;
  constexpr int kWarps = kSelThreads / 32;

  for (int c0 = c_begin + warp * U; c0 < c_end; c0 += kWarps * U) {
    float lv[U][E];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (c0 + u < c_end) {
        VecLoad<T, E>::load(L + (size_t)(c0 + u) * D, lv[u]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) lv[u][e] = 0.f;
      }
    }
    float v[32];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc = fmaf(qr[g][e], lv[u][e], acc);
        v[u * G + g] = acc;
      }
    rs_step<16>(v, lane & 16, 16);
    rs_step<8>(v, lane & 8, 8);
    rs_step<4>(v, lane & 4, 4);
    rs_step<2>(v, lane & 2, 2);
    rs_step<1>(v, lane & 1, 1);
    float x = v[0];  // = score of chunk c0 + lane / G for head lane % G
#pragma unroll
    for (int o = 1; o < G; o <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    const int c = c0 + lane / G;
    if ((lane % G) == 0 && c < c_end) out[c] = x;
  }

  // last CTA of this (batch, KV head) selects
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int t = atomicAdd(a.counters + p, 1);
    s_last = (t == a.n_slices - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  select_pair<T, D, G>(a, p);
  if (threadIdx.x == 0) a.counters[p] = 0;
}

template <typename T, int D, int G>
cudaError_t launch_typed(const SelectArgs& a, cudaStream_t s) {
  dim3 grid(a.n_slices, a.dm.B * a.dm.H);
  score_select_kernel<T, D, G><<<grid, kSelThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_by_shape(const SelectArgs& a, cudaStream_t s) {
  const int D = a.dm.d, G = a.dm.G;
#define LR_CASE(DD, GG) \
  if (D == DD && G == GG) return launch_typed<T, DD, GG>(a, s);
  LR_CASE(64, 1) LR_CASE(64, 2) LR_CASE(64, 4) LR_CASE(64, 8)
  LR_CASE(128, 1) LR_CASE(128, 2) LR_CASE(128, 4) LR_CASE(128, 8)
#undef LR_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  if (a.dm.dtype == LOWRAM_DTYPE_BF16) return launch_by_shape<__nv_bfloat16>(a, s);
  return launch_by_shape<float>(a, s);
}

}  // namespace lowram
