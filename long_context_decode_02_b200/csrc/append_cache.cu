// Periodic re-compression of the generated suffix (agihunt summary, limitations
// paragraph: long generation keeps the generated suffix dense and compresses it
// periodically). A block of whole chunks, compressed on its own at its true positions,
// is appended after a compressed prefix: every array of the result is the prefix's
// followed by the block's, with the block's residual token indices moved by the
// prefix's token count, its CSR offsets by the prefix's row count, and the larger of
// the two landmark-norm bounds. One grid-stride kernel does all of it; blockIdx.y picks
// the array.
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace lowram {
namespace {

constexpr int kAppendThreads = 256;

// rows of `vec16` 16-byte units: row i of the result from the prefix (i < n_p of every
// group of n_p + n_b rows) or the block
__device__ void copy_rows16(const uint4* pre, const uint4* blk, uint4* dst, size_t groups,
                            size_t n_p, size_t n_b, int vec16) {
  const size_t per = (n_p + n_b) * (size_t)vec16;
  const size_t total = groups * per;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t g = i / per, rem = i % per, row = rem / vec16, v = rem % vec16;
    dst[i] = row < n_p ? pre[(g * n_p + row) * vec16 + v] : blk[(g * n_b + row - n_p) * vec16 + v];
  }
}

__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendArgs a) {
  const Dims& p = a.pre;
  const Dims& q = a.blk;
  const int B = p.B, H = p.H;
  const size_t es = p.dtype == LOWRAM_DTYPE_BF16 ? 2 : 4;
  const size_t gstride = (size_t)gridDim.x * blockDim.x;
  const size_t tid0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int Ncp = p.Nc, Ncb = q.Nc;
  switch (blockIdx.y) {
    case 0:   // coef [B][T][r]
      copy_rows16((const uint4*)a.prefix.coef, (const uint4*)a.block.coef, (uint4*)a.dst.coef,
                  B, p.T, q.T, (int)(p.r * es / 16));
      break;
    case 1:   // landmark [B][H][Nc][d]
      copy_rows16((const uint4*)a.prefix.landmark, (const uint4*)a.block.landmark,
                  (uint4*)a.dst.landmark, (size_t)B * H, Ncp, Ncb, (int)(p.d * es / 16));
      break;
    case 2:   // res_val [B][H][n_res][d] (int4: d/2 bytes per row)
      if (p.n_res + q.n_res > 0)
        copy_rows16((const uint4*)a.prefix.res_val, (const uint4*)a.block.res_val,
                    (uint4*)a.dst.res_val, (size_t)B * H, p.n_res, q.n_res,
                    (int)((p.res_int4 ? p.d / 2 : p.d * es) / 16));
      break;
    case 3: {   // res_idx [B][H][n_res]: the block's token indices moved by the prefix's T
      const size_t n = (size_t)p.n_res + q.n_res, total = (size_t)B * H * n;
      for (size_t i = tid0; i < total; i += gstride) {
        const size_t g = i / n, row = i % n;
        a.dst.res_idx[i] = row < (size_t)p.n_res
                               ? a.prefix.res_idx[g * p.n_res + row]
                               : a.block.res_idx[g * q.n_res + row - p.n_res] + p.T;
      }
      break;
    }
    case 4: {   // chunk_ptr [B][H][Nc+1]: the block's offsets moved by the prefix's rows
      const size_t n = (size_t)Ncp + Ncb + 1, total = (size_t)B * H * n;
      for (size_t i = tid0; i < total; i += gstride) {
        const size_t g = i / n, c = i % n;
        a.dst.chunk_ptr[i] = c < (size_t)Ncp
                                 ? a.prefix.chunk_ptr[g * (Ncp + 1) + c]
                                 : a.block.chunk_ptr[g * (Ncb + 1) + c - Ncp] + p.n_res;
      }
      break;
    }
    case 5:   // landmark_norm [B][H]: the larger bound
      for (size_t i = tid0; i < (size_t)B * H; i += gstride)
        a.dst.landmark_norm[i] = fmaxf(a.prefix.landmark_norm[i], a.block.landmark_norm[i]);
      break;
    case 6: {   // chunk positions: written when the result keeps them, checked otherwise
      const size_t n = (size_t)Ncp + Ncb, total = (size_t)B * n;
      for (size_t i = tid0; i < total; i += gstride) {
        const size_t b = i / n, c = i % n;
        int pos;
        if (c < (size_t)Ncp)
          pos = a.prefix.chunk_pos ? a.prefix.chunk_pos[b * Ncp + c] : (int)c;
        else
          pos = a.block.chunk_pos[b * Ncb + c - Ncp];
        if (a.dst.chunk_pos)
          a.dst.chunk_pos[i] = pos;
        else if (pos != (int)c)
          raise_status(a.status, kStatusDeviceCheck);
      }
      break;
    }
    case 7: {   // res_scale [B][H][n_res][d/32] fp16 (int4 rows)
      if (!p.res_int4) break;
      const size_t per = (size_t)p.d / kInt4Group, n = (size_t)p.n_res + q.n_res;
      const size_t total = (size_t)B * H * n * per;
      const __half* ps = (const __half*)a.prefix.res_scale;
      const __half* bs = (const __half*)a.block.res_scale;
      __half* ds = (__half*)a.dst.res_scale;
      for (size_t i = tid0; i < total; i += gstride) {
        const size_t g = i / (n * per), rem = i % (n * per), row = rem / per, e = rem % per;
        ds[i] = row < (size_t)p.n_res ? ps[(g * p.n_res + row) * per + e]
                                      : bs[(g * q.n_res + row - p.n_res) * per + e];
      }
      break;
    }
    default:
      break;
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, int num_sms, cudaStream_t s) {
  append_kernel<<<dim3((unsigned)(num_sms * 4), 8), kAppendThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace lowram
