// Internal declarations of liblowram: launch argument blocks and launchers.
// Not part of the public ABI (include/lowram.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "lowram.h"

namespace lowram {

// Status-word bits set by kernels (read back by lowram_last_error).
constexpr int kStatusDeviceCheck = 1;
constexpr int kStatusTimeout = 2;

// Two-level RoPE tables, position-major (the d/2 pairs of one position are contiguous,
// so a thread rotating one token reads them with vector loads). For pair i, position t:
//   lo[(t & (kRopeLo-1)) * half + i] = (cos, sin)((t mod kRopeLo) * theta_i)
//   hi[(t >> kRopeLoBits) * half + i] = (cos, sin)((t - t mod kRopeLo) * theta_i)
// and the angle of t is recovered by the angle-addition formulas. Entries are computed
// in fp64 on the host, so the fp32 copy carries only its own rounding.
constexpr int kRopeLoBits = 9;
constexpr int kRopeLo = 1 << kRopeLoBits;

struct RopeTables {
  const float2* lo32;
  const float2* hi32;
  const double2* lo64;
  const double2* hi64;
  int n_hi;
  int half;   // d / 2
  const double* theta64;  // theta_i = theta^(-2i/d), i < d/2 (fp64)
  // chunk-base rotations: chunk32[c * half + i] = (cos, sin)(c C theta_i), c < T / C,
  // from fp64 on the host
  const float2* chunk32;
};

struct Dims {
  int B, T, H, Hq, G, d, r, C, F, Nc, k, n_res, act, dtype;
  int P;          // RoPE positions of the original prefix (T unless chunks were evicted)
  int res_int4;   // residual rows stored as int4 codes + fp16 scales per 32 elements
};

// Pair (b, h)'s selection is published by bit b % 32 of word ready_word(dm, b, h) of the
// context's readiness array: H * ceil(B / 32) words, one run per KV head, so one read
// tells the reader of a head every batch element published so far.
__host__ __device__ inline int ready_words_per_head(const Dims& dm) { return (dm.B + 31) / 32; }
__host__ __device__ inline int ready_word(const Dims& dm, int b, int h) {
  return h * ready_words_per_head(dm) + (b >> 5);
}

constexpr int kInt4Group = 32;

// ---------------- decode: landmark scoring + top-k selection ----------------
struct SelectArgs {
  Dims dm;
  const void* landmark;   // [B][H][Nc][d]
  const void* q;          // [B][Hq][d]
  float* scores;          // ctx [B*H][Nc], all bits set between launches
  const float* landmark_norm;  // cache [B*H]: bound of the largest |L|_2 of each pair
  double* cand_s64;       // ws [B*H][Nc]
  int* cand_idx;          // ws [B*H][Nc]
  uint8_t* flags;         // ws [B*H][Nc]
  int* counters;          // ctx [4]: work, exit and pair counters, zero between launches
  int32_t* sel;           // [B*H][k]
  int* ready;             // ctx or null: readiness words, see ready_word()
  int* status;
};
cudaError_t launch_select(const SelectArgs& a, int num_sms, cudaStream_t s);
// landmark_norm[p] = max_c |landmark[p][c]|_2 rounded up to fp32 (fp64 sums).
cudaError_t launch_landmark_norms(const Dims& dm, const void* landmark, float* norm,
                                  cudaStream_t s);
// Stages of landmark rows per (b, h) in the selection kernel: a stage is
// min(65536 / row bytes, 256) rows.
__host__ __device__ inline int select_stages_per_pair(const Dims& dm) {
  const int row_bytes = dm.d * (dm.dtype == LOWRAM_DTYPE_BF16 ? 2 : 4);
  int rows = 65536 / row_bytes;
  if (rows > 256) rows = 256;
  return (dm.Nc + rows - 1) / rows;
}

// ---------------- decode: reconstruct + attend ----------------
struct AttendArgs {
  Dims dm;
  const void* coef;       // [B][T][r]
  const int32_t* res_idx; // [B][H][n_res]
  const void* res_val;    // [B][H][n_res][d]
  const int32_t* chunk_ptr; // [B][H][Nc+1]
  const int32_t* chunk_pos; // [B][Nc] original chunk index of each stored chunk, or null
  const void* res_scale;  // [B][H][n_res][d/32] fp16 (int4 residual rows), or null
  const void* basis;      // [H*d][r]
  const void* w1; const void* b1; const void* w2; const void* b2;
  const void* q;          // [B][Hq][d]
  void* out;              // [B][Hq][d]
  const int32_t* sel;     // [B*H][k]
  float* part;            // ws partials
  RopeTables rope;
  int* status;
  int n_tiles;            // tiles per (b, h)
  int tile_tokens;
  int* ready;             // ctx or null: readiness words (ready_word()); combine clears them
  int wait_ready;         // 1: launched as a programmatic dependent of the selection
                          // kernel; wait for ready[pair] before reading its selection
  int* item_ctr;          // ctx [H]: next tile of each KV head (tcgen05 kernel); combine
                          // clears them
  // decode with a suffix: the combine writes the normalised output in fp32 and the
  // softmax (max in natural-log units, sum) of each query head instead of out; null
  // otherwise
  float* out_f32;         // [B][Hq][d]
  float* out_ml;          // [B][Hq][2]
  // test only (lowram_debug_reconstruct), null otherwise: rebuilt rows of the selected
  // chunks in selection order, row = (b*H + h)*k*C + slot*C + j (j = token in chunk):
  float* dbg_k;           // [rows][d]  K~_rot, as epilogue part A holds it
  float* dbg_h;           // [rows][F]  act(W1 K~_pre + b1), as epilogue part B holds it
  float* dbg_v;           // [rows][d]  the residual row of each token (0 if none); the
                          //            debug value kernel adds W2 h + b2
};
size_t attend_simt_part_floats(const Dims& dm, int n_tiles);
int attend_simt_tile_tokens(const Dims& dm);
cudaError_t launch_attend_simt(const AttendArgs& a, cudaStream_t s);

bool attend_tc_supported(const Dims& dm);
// residual-sum slots in a tcgen05 partial (one per half of the residual rows)
constexpr int kTcResSlots = 2;
size_t attend_tc_part_floats(const Dims& dm, int n_tiles);
constexpr int kTcTileTokens = 128;
cudaError_t launch_attend_tc(const AttendArgs& a, int num_sms, cudaStream_t s);

cudaError_t launch_combine(const AttendArgs& a, bool reorder_form, cudaStream_t s);
// test only: dbg_v[row] += W2_h dbg_h[row] + b2_h for every row of a.dbg_h
cudaError_t launch_debug_values(const AttendArgs& a, cudaStream_t s);

// ---------------- eviction ----------------
// keep the T / C chunks (of P / C) with the largest all-head landmark norm per batch
// element; gather their keys and values; chunk_pos ascending
size_t evict_workspace_bytes(const Dims& dm);
cudaError_t launch_evict(const Dims& dm, const void* k_full, const void* v_full, void* k_kept,
                         void* v_kept, int32_t* chunk_pos, void* ws, cudaStream_t s);

// ---------------- basis fit (randomised range finder, Cholesky-QR) ----------------
size_t fit_basis_workspace_bytes(const Dims& dm, int l);
cudaError_t launch_fit_basis(const Dims& dm, const void* const* k_layers, int n_layers,
                             const double* omega, int l, int n_power, void* basis_out,
                             const RopeTables& rope, int* status, void* ws, cudaStream_t s);

// ---------------- uncompressed baseline ----------------
bool dense_supported(const Dims& dm);
size_t dense_workspace_bytes(const Dims& dm);
cudaError_t launch_dense_decode(const Dims& dm, const void* k, const void* v, const void* q,
                                void* out, void* ws, int* status, cudaStream_t s);
// attention over an uncompressed suffix ([B][s_max][H][d], first n_suffix rows valid),
// merged with the compressed prefix's normalised fp32 output and its softmax (max, sum)
size_t suffix_workspace_bytes(const Dims& dm, int s_max);
cudaError_t launch_suffix_merge(const Dims& dm, const void* k_suffix, const void* v_suffix,
                                int s_max, int n_suffix, const void* q, const float* pre_out,
                                const float* pre_ml, void* out, void* ws, int* status,
                                cudaStream_t s);

// ---------------- encode ----------------
struct EncodeArgs {
  Dims dm;
  const void* k_cache;    // [B][T][H][d]
  const void* v;          // [B][T][H][d]
  const void* basis; const void* w1; const void* b1; const void* w2; const void* b2;
  void* coef; void* landmark; int32_t* res_idx; void* res_val; int32_t* chunk_ptr;
  const int32_t* chunk_pos; // cache [B][Nc] original chunk of each stored chunk, or null
  void* res_scale;        // cache [B][H][n_res][d/32] fp16 (int4 residual rows), or null
  float* err;             // ws [B*H][T]
  double* cand_e64;       // ws [B*H][T]
  int* cand_idx;          // ws [B*H][T]
  uint8_t* flags;         // ws [B*H][T]
  int* cand_count;        // ws [B*H]
  int* in_count;          // ws [B*H]
  RopeTables rope;
  int* status;
  // tensor-core path (encode_tc_supported), else null
  float* c_ws;            // ws [B*T][r] fp32: the unrounded coefficients
  void* basis_t;          // ws [r][H*d] bf16: the basis transposed
  int num_sms;
};
cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s);
bool encode_tc_supported(const Dims& dm);
cudaError_t launch_encode_project_tc(const EncodeArgs& a, void* basis_t, float* c_ws,
                                     int num_sms, cudaStream_t s);
cudaError_t launch_encode_predict_tc(const EncodeArgs& a, const float* c_ws, bool residual_rows,
                                     int num_sms, cudaStream_t s);

// ---------------- periodic re-compression: a compressed block appended ----------------
struct CacheView {   // one cache's arrays (chunk_pos / res_scale null when absent)
  void* coef;
  void* landmark;
  int32_t* res_idx;
  void* res_val;
  int32_t* chunk_ptr;
  float* landmark_norm;
  int32_t* chunk_pos;
  void* res_scale;
};
struct AppendArgs {
  Dims pre, blk;     // the prefix's and the block's dimensions
  CacheView prefix, block, dst;
  int* status;
};
cudaError_t launch_append(const AppendArgs& a, int num_sms, cudaStream_t s);

// 2D tiled TMA map over a row-major [rows][cols] array of dtype (LOWRAM_DTYPE_*), box
// box_rows x box_cols, swizzle 0/32/64/128 bytes; L2 fetches promoted to l2_promo bytes
// (128 or 256). False if the driver refuses it.
bool make_tensor_map_2d(CUtensorMap* m, const void* ptr, int dtype, uint64_t cols,
                        uint64_t rows, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes,
                        int l2_promo = 128);

// Read-only access to a context's configuration and device.
const lowram_config* ctx_config(const lowram_ctx* ctx);
int ctx_device(const lowram_ctx* ctx);

// ---------------- test-only ----------------
cudaError_t launch_debug_tc_tile(const void* a, const void* b, float* d, int k, int mode,
                                 int* status, cudaStream_t s);

}  // namespace lowram
