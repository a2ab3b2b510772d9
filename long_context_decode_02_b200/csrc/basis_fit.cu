// The xKV basis of a layer group by a randomised range finder with Cholesky-QR in place
// of an exact SVD (LowRAM summary on agihunt.info, key paragraph: adjacent layers share
// one SVD basis, computed with a randomised Cholesky-QR that replaces the exact SVD).
//
// The basis is the top-r right singular subspace of A, the group's pre-RoPE key rows
// (every token of every layer, flattened over D = H_kv d), found by subspace iteration on
// A^T A with a random test matrix Omega [D][l] (an input):
//   Y = A^T A Omega;  Q = CholQR2(Y);  n_power times: Q = CholQR2(A^T A Q);
//   Rayleigh-Ritz: S = Q^T A^T A Q = U diag(lambda) U^T;  basis = Q U[:, r leading].
// CholQR2 is Cholesky-QR applied twice: W = Y^T Y = R^T R (R upper), Q = Y R^-1.
//
// Everything is fp64. A^T A is formed once as the Gram matrix G [D][D] (the rows' keys
// are inverse-rotated on the fly with the fp64 RoPE tables), so every later product is
// a small dense one. The eigenproblem of the l x l matrix S is solved by cyclic Jacobi
// rotations in the parallel round-robin order (l/2 disjoint rotations per round).
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace lowram {
namespace {

constexpr int kGB = 64;        // Gram output block
constexpr int kGK = 16;        // rows per k-step
constexpr int kGThreads = 256;
constexpr int kMaxSweeps = 40;

struct FitArgs {
  Dims dm;
  const void* k[8];      // the group's layers: [B][T][H][d] post-RoPE keys
  int n_layers;
  int rows_per_split;
  RopeTables rope;
  double* G;             // [D][D]
  int* status;
};

// element (row t of the layer, column col of D) of the pre-RoPE key: the inverse rotation
// pairs dims (i, i + d/2) of each head
template <typename T>
__device__ __forceinline__ double kpre_elem(const FitArgs& a, const T* k, int row, int col) {
  const Dims& dm = a.dm;
  const int b = row / dm.T, t = row % dm.T;
  const int h = col / dm.d, e = col % dm.d, half = dm.d / 2;
  const int i = e % half;
  const T* base = k + (((size_t)b * dm.T + t) * dm.H + h) * dm.d;
  const double x = ldd(base, i), y = ldd(base, i + half);
  const double2 cs = rope_cs64(a.rope, i, token_position(dm, nullptr, b, t, nullptr));
  return e < half ? x * cs.x + y * cs.y : y * cs.x - x * cs.y;
}

// G[bi*64 .., bj*64 ..] += sum over this CTA's rows of kpre[row][i] kpre[row][j]
template <typename T>
__global__ void __launch_bounds__(kGThreads) gram_kernel(const FitArgs a) {
  const Dims& dm = a.dm;
  const int D = dm.H * dm.d, nbl = D / kGB;
  const int bi = blockIdx.x / nbl, bj = blockIdx.x % nbl;
  const int layer = blockIdx.z;
  const T* k = (const T*)a.k[layer];
  const int n_rows = dm.B * dm.T;
  const int r0 = blockIdx.y * a.rows_per_split;
  const int r1 = min(n_rows, r0 + a.rows_per_split);
  __shared__ double sa[kGK][kGB], sb[kGK][kGB];
  const int tid = threadIdx.x, ti = tid / 16, tj = tid % 16;   // 4 x 4 outputs each
  double acc[4][4];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] = 0.0;
  for (int rb = r0; rb < r1; rb += kGK) {
    __syncthreads();
    for (int o = tid; o < kGK * kGB; o += kGThreads) {
      const int rr = o / kGB, c = o % kGB;
      const int row = rb + rr;
      const bool in = row < r1;
      sa[rr][c] = in ? kpre_elem(a, k, row, bi * kGB + c) : 0.0;
      sb[rr][c] = in ? kpre_elem(a, k, row, bj * kGB + c) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int rr = 0; rr < kGK; ++rr) {
      double va[4], vb[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        va[x] = sa[rr][ti + 16 * x];
        vb[x] = sb[rr][tj + 16 * x];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fma(va[x], vb[y], acc[x][y]);
    }
  }
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y)
      atomicAdd(a.G + (size_t)(bi * kGB + ti + 16 * x) * D + bj * kGB + tj + 16 * y, acc[x][y]);
}

// Y[D][l] = M[D][D] X[D][l] (lda = D); one thread per output, 32 x 8 tiles
__global__ void __launch_bounds__(256) matmul_kernel(const double* M, const double* X, double* Y,
                                                     int n, int kdim, int l) {
  // Y[i][j] = sum_k M[i][k] X[k][j], i < n, j < l
  __shared__ double sm[32][33], sx[32][33];
  const int i0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;   // ty 0..7: rows ty + 8 m
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int k0 = 0; k0 < kdim; k0 += 32) {
    __syncthreads();
    for (int m = 0; m < 4; ++m) {
      const int r = ty + 8 * m;
      sm[r][tx] = (i0 + r < n && k0 + tx < kdim) ? M[(size_t)(i0 + r) * kdim + k0 + tx] : 0.0;
      sx[r][tx] = (k0 + r < kdim && j0 + tx < l) ? X[(size_t)(k0 + r) * l + j0 + tx] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const double xv = sx[kk][tx];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = fma(sm[ty + 8 * m][kk], xv, acc[m]);
    }
  }
  for (int m = 0; m < 4; ++m) {
    const int r = i0 + ty + 8 * m;
    if (r < n && j0 + tx < l) Y[(size_t)r * l + j0 + tx] = acc[m];
  }
}

// W[l][l] = X1^T X2 over n rows (X1, X2 [n][l])
__global__ void __launch_bounds__(256) crossprod_kernel(const double* X1, const double* X2,
                                                        double* W, int n, int l) {
  __shared__ double s1[32][33], s2[32][33];
  const int i0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int k0 = 0; k0 < n; k0 += 32) {
    __syncthreads();
    for (int m = 0; m < 4; ++m) {
      const int r = ty + 8 * m;   // row k0 + r of X
      s1[r][tx] = (k0 + r < n && i0 + tx < l) ? X1[(size_t)(k0 + r) * l + i0 + tx] : 0.0;
      s2[r][tx] = (k0 + r < n && j0 + tx < l) ? X2[(size_t)(k0 + r) * l + j0 + tx] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const double v2 = s2[kk][tx];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = fma(s1[kk][ty + 8 * m], v2, acc[m]);
    }
  }
  for (int m = 0; m < 4; ++m) {
    const int i = i0 + ty + 8 * m, j = j0 + tx;
    if (i < l && j < l) W[(size_t)i * l + j] = acc[m];
  }
}

// In place on W [l][l] (symmetric positive definite): the upper Cholesky factor R
// (W = R^T R), then Rinv = R^-1 (upper) into Ri. One CTA. A non-positive pivot (the
// columns of Y are not of full rank) is reported and the factor replaced by identity.
__global__ void __launch_bounds__(1024) chol_inv_kernel(double* W, double* Ri, int l,
                                                        int* status) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int kk = 0; kk < l; ++kk) {
    if (threadIdx.x == 0) {
      const double p = W[(size_t)kk * l + kk];
      if (!(p > 0.0)) bad = 1;
      W[(size_t)kk * l + kk] = p > 0.0 ? sqrt(p) : 1.0;
    }
    __syncthreads();
    const double piv = W[(size_t)kk * l + kk];
    for (int j = kk + 1 + threadIdx.x; j < l; j += blockDim.x) W[(size_t)kk * l + j] /= piv;
    __syncthreads();
    // trailing update of the upper triangle: W_ij -= R_ki R_kj, kk < i <= j
    const int m = l - kk - 1;
    for (int o = threadIdx.x; o < m * m; o += blockDim.x) {
      const int i = kk + 1 + o / m, j = kk + 1 + o % m;
      if (j >= i) W[(size_t)i * l + j] -= W[(size_t)kk * l + i] * W[(size_t)kk * l + j];
    }
    __syncthreads();
  }
  // Rinv column j: back substitution R x = e_j
  for (int j = threadIdx.x; j < l; j += blockDim.x) {
    for (int i = l - 1; i >= 0; --i) {
      double v = i == j ? 1.0 : 0.0;
      if (i > j) {
        Ri[(size_t)i * l + j] = 0.0;
        continue;
      }
      for (int q = i + 1; q <= j; ++q) v -= W[(size_t)i * l + q] * Ri[(size_t)q * l + j];
      Ri[(size_t)i * l + j] = v / W[(size_t)i * l + i];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && bad) raise_status(status, kStatusDeviceCheck);
}

// Eigen-decomposition of the symmetric S [l][l] by cyclic Jacobi rotations, round-robin
// order (the l/2 rotations of a round touch disjoint index pairs, so one round applies
// them all to the columns, then to the rows). V [l][l] starts as identity and collects the
// rotations; on return diag(S) holds the eigenvalues and the columns of V the vectors.
__global__ void __launch_bounds__(1024) jacobi_kernel(double* S, double* V, int l) {
  const int lp = l + (l & 1);   // an odd size gets a dummy index that pairs with no one
  __shared__ double cs_c[128], cs_s[128];
  __shared__ int pr_p[128], pr_q[128];
  __shared__ double red[32];
  __shared__ int done;
  for (int o = threadIdx.x; o < l * l; o += blockDim.x) V[o] = (o / l == o % l) ? 1.0 : 0.0;
  __syncthreads();
  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    // convergence: off-diagonal mass against the diagonal
    double off = 0.0, dia = 0.0;
    for (int o = threadIdx.x; o < l * l; o += blockDim.x) {
      const double v = S[o];
      if (o / l == o % l) dia += v * v; else off += v * v;
    }
    for (int w = 16; w > 0; w >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, w);
      dia += __shfl_xor_sync(0xffffffffu, dia, w);
    }
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = off;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
      red[0] = t;
    }
    __syncthreads();
    off = red[0];
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dia;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
      done = off <= 1e-30 * t;
    }
    __syncthreads();
    if (done) break;
    for (int round = 0; round < lp - 1; ++round) {
      // pairs of this round (circle method: index 0 fixed, the others rotate)
      for (int i = threadIdx.x; i < lp / 2; i += blockDim.x) {
        auto at = [&](int pos) { return pos == 0 ? 0 : 1 + (pos - 1 + round) % (lp - 1); };
        int p = at(i), q = at(lp - 1 - i);
        if (p > q) { const int t = p; p = q; q = t; }
        double c = 1.0, s = 0.0;
        if (q < l) {
          const double apq = S[(size_t)p * l + q];
          if (apq != 0.0) {
            const double tau = (S[(size_t)q * l + q] - S[(size_t)p * l + p]) / (2.0 * apq);
            const double t = tau >= 0.0 ? 1.0 / (tau + sqrt(1.0 + tau * tau))
                                        : -1.0 / (-tau + sqrt(1.0 + tau * tau));
            c = 1.0 / sqrt(1.0 + t * t);
            s = t * c;
          }
        }
        pr_p[i] = p;
        pr_q[i] = q;
        cs_c[i] = c;
        cs_s[i] = s;
      }
      __syncthreads();
      // columns of S and V: col_p' = c col_p - s col_q, col_q' = s col_p + c col_q
      for (int o = threadIdx.x; o < (lp / 2) * l; o += blockDim.x) {
        const int i = o / l, r = o % l;
        const int p = pr_p[i], q = pr_q[i];
        if (q >= l) continue;
        const double c = cs_c[i], s = cs_s[i];
        const double sp = S[(size_t)r * l + p], sq = S[(size_t)r * l + q];
        S[(size_t)r * l + p] = c * sp - s * sq;
        S[(size_t)r * l + q] = s * sp + c * sq;
        const double vp = V[(size_t)r * l + p], vq = V[(size_t)r * l + q];
        V[(size_t)r * l + p] = c * vp - s * vq;
        V[(size_t)r * l + q] = s * vp + c * vq;
      }
      __syncthreads();
      // rows of S: row_p' = c row_p - s row_q, row_q' = s row_p + c row_q
      for (int o = threadIdx.x; o < (lp / 2) * l; o += blockDim.x) {
        const int i = o / l, cidx = o % l;
        const int p = pr_p[i], q = pr_q[i];
        if (q >= l) continue;
        const double c = cs_c[i], s = cs_s[i];
        const double sp = S[(size_t)p * l + cidx], sq = S[(size_t)q * l + cidx];
        S[(size_t)p * l + cidx] = c * sp - s * sq;
        S[(size_t)q * l + cidx] = s * sp + c * sq;
      }
      __syncthreads();
    }
  }
}

// order[j] = index of the j-th largest eigenvalue (ties to the lower index); one CTA
__global__ void eig_order_kernel(const double* S, int l, int* order) {
  for (int i = threadIdx.x; i < l; i += blockDim.x) {
    const double v = S[(size_t)i * l + i];
    int rank = 0;
    for (int j = 0; j < l; ++j) {
      const double u = S[(size_t)j * l + j];
      rank += (u > v) || (u == v && j < i);
    }
    order[rank] = i;
  }
}

// basis[k][j] = sum_m Q[k][m] V[m][order[j]], j < r, stored in the cache dtype
template <typename T>
__global__ void basis_out_kernel(const double* Q, const double* V, const int* order, T* out,
                                 int D, int l, int r) {
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= D * r) return;
  const int k = o / r, j = o % r, col = order[j];
  double acc = 0.0;
  for (int m = 0; m < l; ++m) acc = fma(Q[(size_t)k * l + m], V[(size_t)m * l + col], acc);
  out[o] = from_f<T>((float)acc);
}

struct FitWs {
  size_t G, Y, Q, Z, W, Ri, S, V, order, total;
};
FitWs fit_ws(const Dims& dm, int l) {
  const size_t D = (size_t)dm.H * dm.d;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  FitWs w{};
  size_t o = 0;
  w.G = o; o = up(o + D * D * 8);
  w.Y = o; o = up(o + D * l * 8);
  w.Q = o; o = up(o + D * l * 8);
  w.Z = o; o = up(o + D * l * 8);
  w.W = o; o = up(o + (size_t)l * l * 8);
  w.Ri = o; o = up(o + (size_t)l * l * 8);
  w.S = o; o = up(o + (size_t)l * l * 8);
  w.V = o; o = up(o + (size_t)l * l * 8);
  w.order = o; o = up(o + (size_t)l * 4);
  w.total = o;
  return w;
}

}  // namespace

size_t fit_basis_workspace_bytes(const Dims& dm, int l) { return fit_ws(dm, l).total; }

cudaError_t launch_fit_basis(const Dims& dm, const void* const* k_layers, int n_layers,
                             const double* omega, int l, int n_power, void* basis_out,
                             const RopeTables& rope, int* status, void* ws, cudaStream_t s) {
  const FitWs w = fit_ws(dm, l);
  uint8_t* base = static_cast<uint8_t*>(ws);
  double* G = reinterpret_cast<double*>(base + w.G);
  double* Y = reinterpret_cast<double*>(base + w.Y);
  double* Q = reinterpret_cast<double*>(base + w.Q);
  double* Z = reinterpret_cast<double*>(base + w.Z);
  double* W = reinterpret_cast<double*>(base + w.W);
  double* Ri = reinterpret_cast<double*>(base + w.Ri);
  double* S = reinterpret_cast<double*>(base + w.S);
  double* V = reinterpret_cast<double*>(base + w.V);
  int* order = reinterpret_cast<int*>(base + w.order);
  const int D = dm.H * dm.d;
  cudaError_t e = cudaMemsetAsync(G, 0, (size_t)D * D * 8, s);
  if (e != cudaSuccess) return e;
  FitArgs a{};
  a.dm = dm;
  for (int i = 0; i < n_layers; ++i) a.k[i] = k_layers[i];
  a.n_layers = n_layers;
  a.rope = rope;
  a.G = G;
  a.status = status;
  const int n_rows = dm.B * dm.T;
  const int nbl = D / kGB;
  // enough row splits to fill the GPU a few times over
  int splits = (4 * 148 + nbl * nbl * n_layers - 1) / (nbl * nbl * n_layers);
  if (splits < 1) splits = 1;
  a.rows_per_split = ((n_rows + splits - 1) / splits + kGK - 1) / kGK * kGK;
  splits = (n_rows + a.rows_per_split - 1) / a.rows_per_split;
  const dim3 gg(nbl * nbl, splits, n_layers);
  if (dm.dtype == LOWRAM_DTYPE_BF16) gram_kernel<__nv_bfloat16><<<gg, kGThreads, 0, s>>>(a);
  else gram_kernel<float><<<gg, kGThreads, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const dim3 mg((D + 31) / 32, (l + 31) / 32), cg((l + 31) / 32, (l + 31) / 32);
  auto cholqr = [&](double* Yin, double* Qout) -> cudaError_t {
    // Qout = Yin R^-1 with Yin^T Yin = R^T R
    crossprod_kernel<<<cg, 256, 0, s>>>(Yin, Yin, W, D, l);
    chol_inv_kernel<<<1, 1024, 0, s>>>(W, Ri, l, status);
    matmul_kernel<<<mg, 256, 0, s>>>(Yin, Ri, Qout, D, l, l);
    return cudaGetLastError();
  };
  auto cholqr2 = [&](double* Yin, double* Qout) -> cudaError_t {
    cudaError_t r = cholqr(Yin, Z);
    if (r == cudaSuccess) r = cholqr(Z, Qout);
    return r;
  };
  matmul_kernel<<<mg, 256, 0, s>>>(G, omega, Y, D, D, l);
  if ((e = cholqr2(Y, Q)) != cudaSuccess) return e;
  for (int it = 0; it < n_power; ++it) {
    matmul_kernel<<<mg, 256, 0, s>>>(G, Q, Y, D, D, l);
    if ((e = cholqr2(Y, Q)) != cudaSuccess) return e;
  }
  // Rayleigh-Ritz: S = Q^T G Q, its eigenvectors by decreasing eigenvalue
  matmul_kernel<<<mg, 256, 0, s>>>(G, Q, Y, D, D, l);
  crossprod_kernel<<<cg, 256, 0, s>>>(Q, Y, S, D, l);
  jacobi_kernel<<<1, 1024, 0, s>>>(S, V, l);
  eig_order_kernel<<<1, 256, 0, s>>>(S, l, order);
  const int n_out = D * dm.r;
  if (dm.dtype == LOWRAM_DTYPE_BF16)
    basis_out_kernel<__nv_bfloat16><<<(n_out + 255) / 256, 256, 0, s>>>(
        Q, V, order, (__nv_bfloat16*)basis_out, D, l, dm.r);
  else
    basis_out_kernel<float><<<(n_out + 255) / 256, 256, 0, s>>>(Q, V, order, (float*)basis_out,
                                                              D, l, dm.r);
  return cudaGetLastError();
}

}  // namespace lowram
