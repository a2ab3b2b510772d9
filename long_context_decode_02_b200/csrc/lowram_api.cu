// Host side of the C ABI declared in include/lowram.h: argument validation, the context
// (RoPE tables, status word, completion counters), cache/workspace layouts, and the
// launch sequences of encode and decode.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "lowram_internal.h"

using namespace lowram;

struct lowram_ctx {
  lowram_config cfg;
  int device;
  int num_sms;
  float2* lo32;
  float2* hi32;
  double2* lo64;
  double2* hi64;
  int n_hi;
  int* status;    // device word
  int* counters;  // device [4]: the selection kernel's work, exit and pair counters
  float* scores;   // device [B*H][Nc], all bits set between launches
  int* ready;     // device [B*H] ints (H * ceil(B/32) used): readiness words, 0 between steps
  int* item_ctr;  // device [H]: tile counters of the tcgen05 attend kernel, 0 between calls
  double* theta64;  // device [d/2]
  float2* chunk32;  // device [T/C][d/2]: (cos, sin)(c C theta_i)
};

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool pow2_in(int v, int lo, int hi) {
  return v >= lo && v <= hi && (v & (v - 1)) == 0;
}

Dims dims_of(const lowram_config& c) {
  Dims d{};
  d.B = c.batch;
  d.T = c.n_tokens;
  d.H = c.n_kv_heads;
  d.Hq = c.n_q_heads;
  d.G = c.n_q_heads / c.n_kv_heads;
  d.d = c.head_dim;
  d.r = c.rank;
  d.C = c.chunk;
  d.F = c.mlp_hidden;
  d.Nc = c.n_tokens / c.chunk;
  d.k = c.top_k < d.Nc ? c.top_k : d.Nc;
  d.n_res = c.n_res;
  d.act = c.act;
  d.dtype = c.dtype;
  d.P = c.n_positions > 0 ? c.n_positions : c.n_tokens;
  d.res_int4 = c.res_format == LOWRAM_RES_INT4_G32 ? 1 : 0;
  return d;
}

bool evicted(const lowram_config& c) { return c.n_positions > 0 && c.n_positions > c.n_tokens; }

bool use_tc(const lowram_config& c) {
  if (c.decode_variant == LOWRAM_DECODE_SIMT) return false;
  const bool ok = attend_tc_supported(dims_of(c));
  return c.decode_variant == LOWRAM_DECODE_TCGEN05 ? true : ok;
}

int n_tiles_of(const lowram_config& c) {
  const Dims d = dims_of(c);
  const int tt = use_tc(c) ? kTcTileTokens : attend_simt_tile_tokens(d);
  return (d.k * d.C + tt - 1) / tt;
}

size_t elem_size(const lowram_config& c) { return c.dtype == LOWRAM_DTYPE_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Scoped switch of the calling thread's current device.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

struct DecodeWs {
  size_t cand_s64, cand_idx, flags, sel, part, total;
};
DecodeWs decode_ws(const lowram_config& c) {
  const Dims d = dims_of(c);
  const size_t pairs = (size_t)d.B * d.H;
  const int nt = n_tiles_of(c);
  const size_t part_floats = use_tc(c) ? attend_tc_part_floats(d, nt)
                                       : attend_simt_part_floats(d, nt);
  DecodeWs w{};
  size_t o = 0;
  w.cand_s64 = o; o = align_up(o + pairs * d.Nc * sizeof(double));
  w.cand_idx = o; o = align_up(o + pairs * d.Nc * sizeof(int));
  w.flags = o;    o = align_up(o + pairs * d.Nc);
  w.sel = o;      o = align_up(o + pairs * d.k * sizeof(int32_t));
  w.part = o;     o = align_up(o + part_floats * sizeof(float));
  w.total = o;
  return w;
}

struct EncodeWs {
  size_t err, cand_e64, cand_idx, flags, cand_count, in_count, c_ws, basis_t, total;
};
EncodeWs encode_ws(const lowram_config& c) {
  const size_t pairs = (size_t)c.batch * c.n_kv_heads;
  const size_t T = (size_t)c.n_tokens;
  EncodeWs w{};
  size_t o = 0;
  if (encode_tc_supported(dims_of(c))) {   // the tensor-core encode's own arrays
    w.c_ws = o;     o = align_up(o + (size_t)c.batch * T * c.rank * sizeof(float));
    w.basis_t = o;  o = align_up(o + (size_t)c.rank * c.n_kv_heads * c.head_dim * 2);
  }
  w.err = o;        o = align_up(o + pairs * T * sizeof(float));
  w.cand_e64 = o;   o = align_up(o + pairs * T * sizeof(double));
  w.cand_idx = o;   o = align_up(o + pairs * T * sizeof(int));
  w.flags = o;      o = align_up(o + pairs * T);
  w.cand_count = o; o = align_up(o + pairs * sizeof(int));
  w.in_count = o;   o = align_up(o + pairs * sizeof(int));
  w.total = o;
  return w;
}

RopeTables rope_of(const lowram_ctx* ctx) {
  RopeTables r{};
  r.lo32 = ctx->lo32;
  r.hi32 = ctx->hi32;
  r.lo64 = ctx->lo64;
  r.hi64 = ctx->hi64;
  r.n_hi = ctx->n_hi;
  r.half = ctx->cfg.head_dim / 2;
  r.theta64 = ctx->theta64;
  r.chunk32 = ctx->chunk32;
  return r;
}

lowram_status check_layer_params(const lowram_layer_params* p) {
  if (!p || !p->basis || !p->w1 || !p->b1 || !p->w2 || !p->b2) return LOWRAM_ERR_INVALID_ARG;
  if (!aligned16(p->basis) || !aligned16(p->w1) || !aligned16(p->b1) || !aligned16(p->w2) ||
      !aligned16(p->b2))
    return LOWRAM_ERR_ALIGN;
  return LOWRAM_OK;
}

// res_idx / res_val (/ res_scale) may be NULL when the configuration keeps no residual
// rows; chunk_pos is required exactly when chunks were evicted.
lowram_status check_cache(const lowram_cache* c, const lowram_config& cfg) {
  const int n_res = cfg.n_res;
  if (!c || !c->coef || !c->landmark || !c->chunk_ptr || !c->landmark_norm)
    return LOWRAM_ERR_INVALID_ARG;
  if (n_res > 0 && (!c->res_idx || !c->res_val)) return LOWRAM_ERR_INVALID_ARG;
  if (n_res > 0 && cfg.res_format == LOWRAM_RES_INT4_G32 && !c->res_scale)
    return LOWRAM_ERR_INVALID_ARG;
  if (evicted(cfg) && !c->chunk_pos) return LOWRAM_ERR_INVALID_ARG;
  if (!aligned16(c->coef) || !aligned16(c->landmark) || !aligned16(c->res_idx) ||
      !aligned16(c->res_val) || !aligned16(c->chunk_ptr) || !aligned16(c->landmark_norm) ||
      !aligned16(c->chunk_pos) || !aligned16(c->res_scale))
    return LOWRAM_ERR_ALIGN;
  return LOWRAM_OK;
}

// the pointers the kernels see: chunk_pos only with eviction, res_scale only for int4
const int32_t* chunk_pos_of(const lowram_cache* c, const lowram_config& cfg) {
  return evicted(cfg) ? c->chunk_pos : nullptr;
}
const void* res_scale_of(const lowram_cache* c, const lowram_config& cfg) {
  return cfg.res_format == LOWRAM_RES_INT4_G32 ? c->res_scale : nullptr;
}

}  // namespace

extern "C" {

lowram_status lowram_check_config(const lowram_config* c) {
  if (!c) return LOWRAM_ERR_INVALID_ARG;
  if (c->act != LOWRAM_ACT_SILU && c->act != LOWRAM_ACT_GELU_ERF) return LOWRAM_ERR_INVALID_ARG;
  if (c->dtype != LOWRAM_DTYPE_F32 && c->dtype != LOWRAM_DTYPE_BF16) return LOWRAM_ERR_INVALID_ARG;
  if (c->decode_variant < LOWRAM_DECODE_AUTO || c->decode_variant > LOWRAM_DECODE_TCGEN05)
    return LOWRAM_ERR_INVALID_ARG;
  if (c->reserved != 0) return LOWRAM_ERR_INVALID_ARG;
  if (c->res_format != LOWRAM_RES_STORE && c->res_format != LOWRAM_RES_INT4_G32)
    return LOWRAM_ERR_INVALID_ARG;
  if (c->n_positions < 0) return LOWRAM_ERR_SHAPE;
  if (c->n_positions > 0 && (c->n_positions < c->n_tokens || c->chunk < 1 ||
                             c->n_positions % c->chunk != 0))
    return LOWRAM_ERR_SHAPE;
  if (c->n_positions > (1 << 24)) return LOWRAM_ERR_UNSUPPORTED;
  if (!(c->rope_theta > 0.0) || !std::isfinite(c->rope_theta)) return LOWRAM_ERR_INVALID_ARG;
  if (c->batch < 1 || c->n_tokens < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 ||
      c->head_dim < 1 || c->rank < 1 || c->chunk < 1 || c->mlp_hidden < 1)
    return LOWRAM_ERR_SHAPE;
  if (c->n_q_heads % c->n_kv_heads != 0) return LOWRAM_ERR_SHAPE;
  if (c->n_tokens % c->chunk != 0) return LOWRAM_ERR_SHAPE;
  if (c->top_k < 1) return LOWRAM_ERR_SHAPE;
  if (c->n_res < 0 || c->n_res > c->n_tokens) return LOWRAM_ERR_SHAPE;
  if (c->rank > c->n_kv_heads * c->head_dim) return LOWRAM_ERR_SHAPE;
  if (c->head_dim != 64 && c->head_dim != 128) return LOWRAM_ERR_UNSUPPORTED;
  if (c->rank % 16 != 0 || c->rank < 16 || c->rank > 256) return LOWRAM_ERR_UNSUPPORTED;
  if (!pow2_in(c->chunk, 1, 32)) return LOWRAM_ERR_UNSUPPORTED;
  if (c->mlp_hidden != 128 && c->mlp_hidden != 256) return LOWRAM_ERR_UNSUPPORTED;
  if (!pow2_in(c->n_q_heads / c->n_kv_heads, 1, 8)) return LOWRAM_ERR_UNSUPPORTED;
  if (c->n_tokens % 16 != 0 || c->n_tokens > (1 << 24)) return LOWRAM_ERR_UNSUPPORTED;
  if (c->n_kv_heads * c->head_dim > 2048) return LOWRAM_ERR_UNSUPPORTED;
  if ((size_t)c->batch * c->n_kv_heads * (size_t)(c->n_tokens / c->chunk) > ((size_t)1 << 30))
    return LOWRAM_ERR_UNSUPPORTED;   // landmark rows of one call, indexed in 32 bits
  if (c->decode_variant == LOWRAM_DECODE_TCGEN05 && !attend_tc_supported(dims_of(*c)))
    return LOWRAM_ERR_UNSUPPORTED;
  // int4 residual rows are written by the tensor-core encode
  if (c->res_format == LOWRAM_RES_INT4_G32 && !encode_tc_supported(dims_of(*c)))
    return LOWRAM_ERR_UNSUPPORTED;
  return LOWRAM_OK;
}

lowram_status lowram_cache_layout(const lowram_config* c, size_t bytes_out[8]) {
  if (!bytes_out) return LOWRAM_ERR_INVALID_ARG;
  const lowram_status st = lowram_check_config(c);
  if (st != LOWRAM_OK) return st;
  const size_t es = elem_size(*c);
  const size_t B = c->batch, T = c->n_tokens, H = c->n_kv_heads, d = c->head_dim;
  const bool q4 = c->res_format == LOWRAM_RES_INT4_G32;
  bytes_out[0] = B * T * c->rank * es;
  bytes_out[1] = B * H * (T / c->chunk) * d * es;
  bytes_out[2] = B * H * (size_t)c->n_res * sizeof(int32_t);
  bytes_out[3] = B * H * (size_t)c->n_res * (q4 ? d / 2 : d * es);
  bytes_out[4] = B * H * (T / c->chunk + 1) * sizeof(int32_t);
  bytes_out[5] = B * H * sizeof(float);
  bytes_out[6] = evicted(*c) ? B * (T / c->chunk) * sizeof(int32_t) : 0;
  bytes_out[7] = q4 ? B * H * (size_t)c->n_res * (d / kInt4Group) * 2 : 0;
  return LOWRAM_OK;
}

lowram_status lowram_workspace_size(const lowram_config* c, int op, size_t* bytes) {
  if (!bytes) return LOWRAM_ERR_INVALID_ARG;
  const lowram_status st = lowram_check_config(c);
  if (st != LOWRAM_OK) return st;
  if (op == LOWRAM_OP_ENCODE) { *bytes = encode_ws(*c).total; return LOWRAM_OK; }
  if (op == LOWRAM_OP_DECODE) { *bytes = decode_ws(*c).total; return LOWRAM_OK; }
  if (op == LOWRAM_OP_EVICT) {
    if (!evicted(*c)) return LOWRAM_ERR_SHAPE;
    *bytes = evict_workspace_bytes(dims_of(*c));
    return LOWRAM_OK;
  }
  if (op == LOWRAM_OP_DENSE) {
    if (!dense_supported(dims_of(*c))) return LOWRAM_ERR_UNSUPPORTED;
    *bytes = dense_workspace_bytes(dims_of(*c));
    return LOWRAM_OK;
  }
  return LOWRAM_ERR_INVALID_ARG;
}

lowram_status lowram_create(const lowram_config* c, int device, lowram_ctx** out) {
  if (!out) return LOWRAM_ERR_INVALID_ARG;
  const lowram_status st = lowram_check_config(c);
  if (st != LOWRAM_OK) return st;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  DeviceGuard g(device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  lowram_ctx* ctx = new (std::nothrow) lowram_ctx();
  if (!ctx) return LOWRAM_ERR_CUDA;
  ctx->cfg = *c;
  ctx->device = device;
  cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, device);
  const int half = c->head_dim / 2;
  const int n_pos = dims_of(*c).P;   // RoPE positions (the original prefix)
  ctx->n_hi = (n_pos + kRopeLo - 1) / kRopeLo;
  // two-level tables, fp64 on the host: theta_i = theta^(-2i/d)
  std::vector<float2> lo32((size_t)half * kRopeLo), hi32((size_t)half * ctx->n_hi);
  std::vector<double2> lo64((size_t)half * kRopeLo), hi64((size_t)half * ctx->n_hi);
  std::vector<double> th64((size_t)half);
  const size_t n_chunks = (size_t)(n_pos / c->chunk);
  std::vector<float2> chunk32(n_chunks * half);
  for (int i = 0; i < half; ++i) {
    const double th = std::pow(c->rope_theta, -2.0 * i / c->head_dim);
    th64[i] = th;
    for (int t = 0; t < kRopeLo; ++t) {
      const double ang = (double)t * th;
      lo64[(size_t)t * half + i] = make_double2(std::cos(ang), std::sin(ang));
      lo32[(size_t)t * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
    for (int j = 0; j < ctx->n_hi; ++j) {
      const double ang = (double)j * kRopeLo * th;
      hi64[(size_t)j * half + i] = make_double2(std::cos(ang), std::sin(ang));
      hi32[(size_t)j * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
    for (size_t cc = 0; cc < n_chunks; ++cc) {
      const double ang = (double)(cc * (size_t)c->chunk) * th;
      chunk32[cc * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
  }
  const size_t pairs = (size_t)c->batch * c->n_kv_heads;
  bool ok = cudaMalloc(&ctx->lo32, lo32.size() * sizeof(float2)) == cudaSuccess &&
            cudaMalloc(&ctx->hi32, hi32.size() * sizeof(float2)) == cudaSuccess &&
            cudaMalloc(&ctx->lo64, lo64.size() * sizeof(double2)) == cudaSuccess &&
            cudaMalloc(&ctx->hi64, hi64.size() * sizeof(double2)) == cudaSuccess &&
            cudaMalloc(&ctx->status, sizeof(int)) == cudaSuccess &&
            cudaMalloc(&ctx->counters, 4 * sizeof(int)) == cudaSuccess &&
            cudaMalloc(&ctx->ready, pairs * sizeof(int)) == cudaSuccess &&
            cudaMalloc(&ctx->item_ctr, (size_t)c->n_kv_heads * sizeof(int)) == cudaSuccess &&
            cudaMalloc(&ctx->scores, pairs * (size_t)(c->n_tokens / c->chunk) * sizeof(float)) == cudaSuccess &&
            cudaMalloc(&ctx->theta64, th64.size() * sizeof(double)) == cudaSuccess &&
            cudaMalloc(&ctx->chunk32, chunk32.size() * sizeof(float2)) == cudaSuccess;
  ok = ok &&
       cudaMemcpy(ctx->lo32, lo32.data(), lo32.size() * sizeof(float2), cudaMemcpyHostToDevice) == cudaSuccess &&
       cudaMemcpy(ctx->hi32, hi32.data(), hi32.size() * sizeof(float2), cudaMemcpyHostToDevice) == cudaSuccess &&
       cudaMemcpy(ctx->lo64, lo64.data(), lo64.size() * sizeof(double2), cudaMemcpyHostToDevice) == cudaSuccess &&
       cudaMemcpy(ctx->hi64, hi64.data(), hi64.size() * sizeof(double2), cudaMemcpyHostToDevice) == cudaSuccess &&
       cudaMemset(ctx->status, 0, sizeof(int)) == cudaSuccess &&
       cudaMemset(ctx->counters, 0, 4 * sizeof(int)) == cudaSuccess &&
       cudaMemset(ctx->ready, 0, pairs * sizeof(int)) == cudaSuccess &&
       cudaMemset(ctx->item_ctr, 0, (size_t)c->n_kv_heads * sizeof(int)) == cudaSuccess &&
       cudaMemset(ctx->scores, 0xff, pairs * (size_t)(c->n_tokens / c->chunk) * sizeof(float)) == cudaSuccess &&
       cudaMemcpy(ctx->theta64, th64.data(), th64.size() * sizeof(double), cudaMemcpyHostToDevice) == cudaSuccess &&
       cudaMemcpy(ctx->chunk32, chunk32.data(), chunk32.size() * sizeof(float2), cudaMemcpyHostToDevice) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    lowram_destroy(ctx);
    return LOWRAM_ERR_CUDA;
  }
  *out = ctx;
  return LOWRAM_OK;
}

void lowram_destroy(lowram_ctx* ctx) {
  if (!ctx) return;
  DeviceGuard g(ctx->device);
  cudaFree(ctx->lo32);
  cudaFree(ctx->hi32);
  cudaFree(ctx->lo64);
  cudaFree(ctx->hi64);
  cudaFree(ctx->status);
  cudaFree(ctx->counters);
  cudaFree(ctx->scores);
  cudaFree(ctx->ready);
  cudaFree(ctx->item_ctr);
  cudaFree(ctx->theta64);
  cudaFree(ctx->chunk32);
  delete ctx;
}

lowram_status lowram_encode(lowram_ctx* ctx, const void* k_cache, const void* v,
                            const lowram_layer_params* params, const lowram_cache* out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!ctx || !k_cache || !v || !workspace) return LOWRAM_ERR_INVALID_ARG;
  lowram_status st = check_layer_params(params);
  if (st != LOWRAM_OK) return st;
  if ((st = check_cache(out, ctx->cfg)) != LOWRAM_OK) return st;
  if (!aligned16(k_cache) || !aligned16(v) || !aligned16(workspace)) return LOWRAM_ERR_ALIGN;
  const lowram_config& c = ctx->cfg;
  const EncodeWs w = encode_ws(c);
  if (workspace_bytes < w.total) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  EncodeArgs a{};
  a.dm = dims_of(c);
  a.k_cache = k_cache;
  a.v = v;
  a.basis = params->basis; a.w1 = params->w1; a.b1 = params->b1; a.w2 = params->w2; a.b2 = params->b2;
  a.coef = out->coef; a.landmark = out->landmark; a.res_idx = out->res_idx;
  a.res_val = out->res_val; a.chunk_ptr = out->chunk_ptr;
  a.chunk_pos = chunk_pos_of(out, c);
  a.res_scale = const_cast<void*>(res_scale_of(out, c));
  a.err = reinterpret_cast<float*>(ws + w.err);
  a.cand_e64 = reinterpret_cast<double*>(ws + w.cand_e64);
  a.cand_idx = reinterpret_cast<int*>(ws + w.cand_idx);
  a.flags = ws + w.flags;
  a.cand_count = reinterpret_cast<int*>(ws + w.cand_count);
  a.in_count = reinterpret_cast<int*>(ws + w.in_count);
  a.rope = rope_of(ctx);
  a.status = ctx->status;
  if (encode_tc_supported(a.dm)) {
    a.c_ws = reinterpret_cast<float*>(ws + w.c_ws);
    a.basis_t = ws + w.basis_t;
  }
  a.num_sms = ctx->num_sms;
  cudaError_t e = launch_encode(a, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess)
    e = launch_landmark_norms(dims_of(c), out->landmark, out->landmark_norm,
                              static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) { cudaGetLastError(); return LOWRAM_ERR_CUDA; }
  return LOWRAM_OK;
}

}  // extern "C"

namespace {

lowram_status select_impl(lowram_ctx* ctx, const void* landmark, const float* landmark_norm,
                          const void* q, int32_t* sel,
                          uint8_t* ws, const DecodeWs& w, cudaStream_t s, bool set_ready) {
  const Dims dm = dims_of(ctx->cfg);
  SelectArgs sa{};
  sa.dm = dm;
  sa.landmark = landmark;
  sa.q = q;
  sa.scores = ctx->scores;
  sa.landmark_norm = landmark_norm;
  sa.cand_s64 = reinterpret_cast<double*>(ws + w.cand_s64);
  sa.cand_idx = reinterpret_cast<int*>(ws + w.cand_idx);
  sa.flags = ws + w.flags;
  sa.counters = ctx->counters;
  sa.sel = sel;
  sa.ready = set_ready ? ctx->ready : nullptr;
  sa.status = ctx->status;
  if (launch_select(sa, ctx->num_sms, s) != cudaSuccess) { cudaGetLastError(); return LOWRAM_ERR_CUDA; }
  return LOWRAM_OK;
}

// dbg (test only, else null): {k_rot, h_act, v_rec} rows written by the tcgen05 kernel
lowram_status attend_impl(lowram_ctx* ctx, const lowram_cache* cache,
                          const lowram_layer_params* params, const void* q, const int32_t* sel,
                          void* out, uint8_t* ws, const DecodeWs& w, cudaStream_t s,
                          bool after_select, float* const* dbg = nullptr,
                          float* const* f32 = nullptr) {
  const lowram_config& c = ctx->cfg;
  const Dims dm = dims_of(c);
  AttendArgs aa{};
  aa.dm = dm;
  aa.coef = cache->coef;
  aa.res_idx = cache->res_idx;
  aa.res_val = cache->res_val;
  aa.chunk_ptr = cache->chunk_ptr;
  aa.chunk_pos = chunk_pos_of(cache, c);
  aa.res_scale = res_scale_of(cache, c);
  aa.basis = params->basis; aa.w1 = params->w1; aa.b1 = params->b1; aa.w2 = params->w2; aa.b2 = params->b2;
  aa.q = q;
  aa.out = out;
  aa.sel = sel;
  aa.part = reinterpret_cast<float*>(ws + w.part);
  aa.rope = rope_of(ctx);
  aa.status = ctx->status;
  aa.n_tiles = n_tiles_of(c);
  const bool tc = use_tc(c);
  aa.tile_tokens = tc ? kTcTileTokens : attend_simt_tile_tokens(dm);
  // right after the selection kernel the tcgen05 kernel overlaps its tail, pair by pair
  aa.ready = tc && after_select ? ctx->ready : nullptr;
  aa.wait_ready = aa.ready ? 1 : 0;
  aa.item_ctr = tc ? ctx->item_ctr : nullptr;
  if (f32) {   // decode with a suffix: fp32 output and softmax statistics
    aa.out_f32 = f32[0];
    aa.out_ml = f32[1];
  }
  if (dbg) {
    aa.dbg_k = dbg[0];
    aa.dbg_h = dbg[1];
    aa.dbg_v = dbg[2];
  }
  cudaError_t e = tc ? launch_attend_tc(aa, ctx->num_sms, s) : launch_attend_simt(aa, s);
  if (e == cudaSuccess) e = launch_combine(aa, tc, s);
  if (e == cudaSuccess && dbg) e = launch_debug_values(aa, s);
  if (e != cudaSuccess) { cudaGetLastError(); return LOWRAM_ERR_CUDA; }
  return LOWRAM_OK;
}

}  // namespace

extern "C" {

lowram_status lowram_select_chunks(lowram_ctx* ctx, const void* landmark,
                                   const float* landmark_norm, const void* q, int32_t* sel_out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!ctx || !landmark || !landmark_norm || !q || !sel_out || !workspace)
    return LOWRAM_ERR_INVALID_ARG;
  if (!aligned16(landmark) || !aligned16(landmark_norm) || !aligned16(q) ||
      !aligned16(sel_out) || !aligned16(workspace))
    return LOWRAM_ERR_ALIGN;
  const DecodeWs w = decode_ws(ctx->cfg);
  if (workspace_bytes < w.total) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  return select_impl(ctx, landmark, landmark_norm, q, sel_out,
                     static_cast<uint8_t*>(workspace), w, static_cast<cudaStream_t>(stream),
                     false);
}

lowram_status lowram_landmark_norms(lowram_ctx* ctx, const void* landmark, float* landmark_norm,
                                    void* stream) {
  if (!ctx || !landmark || !landmark_norm) return LOWRAM_ERR_INVALID_ARG;
  if (!aligned16(landmark) || !aligned16(landmark_norm)) return LOWRAM_ERR_ALIGN;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  if (launch_landmark_norms(dims_of(ctx->cfg), landmark, landmark_norm,
                            static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  return LOWRAM_OK;
}

lowram_status lowram_attend_selected(lowram_ctx* ctx, const lowram_cache* cache,
                                     const lowram_layer_params* params, const void* q,
                                     const int32_t* sel, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!ctx || !q || !sel || !out || !workspace) return LOWRAM_ERR_INVALID_ARG;
  lowram_status st = check_layer_params(params);
  if (st != LOWRAM_OK) return st;
  if ((st = check_cache(cache, ctx->cfg)) != LOWRAM_OK) return st;
  if (!aligned16(q) || !aligned16(sel) || !aligned16(out) || !aligned16(workspace))
    return LOWRAM_ERR_ALIGN;
  const DecodeWs w = decode_ws(ctx->cfg);
  if (workspace_bytes < w.total) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  return attend_impl(ctx, cache, params, q, sel, out, static_cast<uint8_t*>(workspace), w,
                     static_cast<cudaStream_t>(stream), false);
}

lowram_status lowram_debug_reconstruct(lowram_ctx* ctx, const lowram_cache* cache,
                                      const lowram_layer_params* params, const void* q,
                                      const int32_t* sel, void* out, float* k_rot,
                                      float* h_act, float* v_rec, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!ctx || !q || !sel || !out || !workspace || !k_rot || !h_act || !v_rec)
    return LOWRAM_ERR_INVALID_ARG;
  lowram_status st = check_layer_params(params);
  if (st != LOWRAM_OK) return st;
  if ((st = check_cache(cache, ctx->cfg)) != LOWRAM_OK) return st;
  if (!aligned16(q) || !aligned16(sel) || !aligned16(out) || !aligned16(workspace) ||
      !aligned16(k_rot) || !aligned16(h_act) || !aligned16(v_rec))
    return LOWRAM_ERR_ALIGN;
  if (!use_tc(ctx->cfg)) return LOWRAM_ERR_UNSUPPORTED;
  const DecodeWs w = decode_ws(ctx->cfg);
  if (workspace_bytes < w.total) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  const Dims dm = dims_of(ctx->cfg);
  const size_t rows = (size_t)dm.B * dm.H * dm.k * dm.C;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(k_rot, 0, rows * dm.d * sizeof(float), s) != cudaSuccess ||
      cudaMemsetAsync(h_act, 0, rows * dm.F * sizeof(float), s) != cudaSuccess ||
      cudaMemsetAsync(v_rec, 0, rows * dm.d * sizeof(float), s) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  float* const dbg[3] = {k_rot, h_act, v_rec};
  return attend_impl(ctx, cache, params, q, sel, out, static_cast<uint8_t*>(workspace), w, s,
                     false, dbg);
}

lowram_status lowram_debug_attend_unpublished(lowram_ctx* ctx, const lowram_cache* cache,
                                              const lowram_layer_params* params, const void* q,
                                              const int32_t* sel, void* out, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  if (!ctx || !q || !sel || !out || !workspace) return LOWRAM_ERR_INVALID_ARG;
  lowram_status st = check_layer_params(params);
  if (st != LOWRAM_OK) return st;
  if ((st = check_cache(cache, ctx->cfg)) != LOWRAM_OK) return st;
  if (!aligned16(q) || !aligned16(sel) || !aligned16(out) || !aligned16(workspace))
    return LOWRAM_ERR_ALIGN;
  if (!use_tc(ctx->cfg)) return LOWRAM_ERR_UNSUPPORTED;
  const DecodeWs w = decode_ws(ctx->cfg);
  if (workspace_bytes < w.total) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  // as right after a selection launch, but none ran: the ready flags stay 0
  return attend_impl(ctx, cache, params, q, sel, out, static_cast<uint8_t*>(workspace), w,
                     static_cast<cudaStream_t>(stream), true);
}

lowram_status lowram_decode_step(lowram_ctx* ctx, const lowram_cache* cache,
                                 const lowram_layer_params* params, const void* q, void* out,
                                 int32_t* sel_out, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!ctx || !q || !out || !workspace) return LOWRAM_ERR_INVALID_ARG;
  lowram_status st = check_layer_params(params);
  if (st != LOWRAM_OK) return st;
  if ((st = check_cache(cache, ctx->cfg)) != LOWRAM_OK) return st;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace) ||
      (sel_out && !aligned16(sel_out)))
    return LOWRAM_ERR_ALIGN;
  const DecodeWs w = decode_ws(ctx->cfg);
  if (workspace_bytes < w.total) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(ws + w.sel);
  const bool tc = use_tc(ctx->cfg);
  if ((st = select_impl(ctx, cache->landmark, cache->landmark_norm, q, sel, ws, w, s, tc)) !=
      LOWRAM_OK)
    return st;
  return attend_impl(ctx, cache, params, q, sel, out, ws, w, s, tc);
}

lowram_status lowram_evict(lowram_ctx* ctx, const void* k_full, const void* v_full,
                           void* k_kept, void* v_kept, int32_t* chunk_pos, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!ctx || !k_full || !v_full || !k_kept || !v_kept || !chunk_pos || !workspace)
    return LOWRAM_ERR_INVALID_ARG;
  if (!aligned16(k_full) || !aligned16(v_full) || !aligned16(k_kept) || !aligned16(v_kept) ||
      !aligned16(chunk_pos) || !aligned16(workspace))
    return LOWRAM_ERR_ALIGN;
  if (!evicted(ctx->cfg)) return LOWRAM_ERR_SHAPE;
  const Dims dm = dims_of(ctx->cfg);
  if (workspace_bytes < evict_workspace_bytes(dm)) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  if (launch_evict(dm, k_full, v_full, k_kept, v_kept, chunk_pos, workspace,
                   static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  return LOWRAM_OK;
}

lowram_status lowram_append(lowram_ctx* dst_ctx, const lowram_cache* dst,
                            const lowram_ctx* prefix_ctx, const lowram_cache* prefix,
                            const lowram_ctx* block_ctx, const lowram_cache* block,
                            void* stream) {
  if (!dst_ctx || !dst || !prefix_ctx || !prefix || !block_ctx || !block)
    return LOWRAM_ERR_INVALID_ARG;
  const lowram_config &cd = dst_ctx->cfg, &cp = prefix_ctx->cfg, &cb = block_ctx->cfg;
  auto same = [](const lowram_config& x, const lowram_config& y) {
    return x.batch == y.batch && x.n_kv_heads == y.n_kv_heads && x.n_q_heads == y.n_q_heads &&
           x.head_dim == y.head_dim && x.rank == y.rank && x.chunk == y.chunk &&
           x.mlp_hidden == y.mlp_hidden && x.act == y.act && x.dtype == y.dtype &&
           x.res_format == y.res_format;
  };
  if (!same(cd, cp) || !same(cd, cb)) return LOWRAM_ERR_SHAPE;
  if (cd.n_tokens != cp.n_tokens + cb.n_tokens || cd.n_res != cp.n_res + cb.n_res)
    return LOWRAM_ERR_SHAPE;
  // the block carries its chunks' positions; a result that keeps positions must cover them
  if (!evicted(cb)) return LOWRAM_ERR_SHAPE;
  if (evicted(cd) && cd.n_positions < cb.n_positions) return LOWRAM_ERR_SHAPE;
  lowram_status st;
  if ((st = check_cache(dst, cd)) != LOWRAM_OK) return st;
  if ((st = check_cache(prefix, cp)) != LOWRAM_OK) return st;
  if ((st = check_cache(block, cb)) != LOWRAM_OK) return st;
  if (prefix_ctx->device != dst_ctx->device || block_ctx->device != dst_ctx->device)
    return LOWRAM_ERR_INVALID_ARG;
  auto view = [](const lowram_cache* c, const lowram_config& cfg) {
    return CacheView{c->coef, c->landmark, c->res_idx, c->res_val, c->chunk_ptr,
                     c->landmark_norm, const_cast<int32_t*>(chunk_pos_of(c, cfg)),
                     const_cast<void*>(res_scale_of(c, cfg))};
  };
  AppendArgs a{};
  a.pre = dims_of(cp);
  a.blk = dims_of(cb);
  a.prefix = view(prefix, cp);
  a.block = view(block, cb);
  a.dst = view(dst, cd);
  a.status = dst_ctx->status;
  DeviceGuard g(dst_ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  if (launch_append(a, dst_ctx->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  return LOWRAM_OK;
}

lowram_status lowram_fit_basis_workspace_size(const lowram_config* c, int32_t l, size_t* bytes) {
  if (!bytes) return LOWRAM_ERR_INVALID_ARG;
  const lowram_status st = lowram_check_config(c);
  if (st != LOWRAM_OK) return st;
  const int D = c->n_kv_heads * c->head_dim;
  if (l < c->rank || l > D || l > 256) return LOWRAM_ERR_SHAPE;
  if (D % 64 != 0) return LOWRAM_ERR_UNSUPPORTED;
  *bytes = fit_basis_workspace_bytes(dims_of(*c), l);
  return LOWRAM_OK;
}

lowram_status lowram_fit_basis(lowram_ctx* ctx, const void* const* k_layers, int32_t n_layers,
                               const double* omega, int32_t l, int32_t n_power,
                               void* basis_out, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (!ctx || !k_layers || !omega || !basis_out || !workspace) return LOWRAM_ERR_INVALID_ARG;
  if (n_layers < 1 || n_layers > 8 || n_power < 0 || n_power > 16) return LOWRAM_ERR_INVALID_ARG;
  for (int i = 0; i < n_layers; ++i) {
    if (!k_layers[i]) return LOWRAM_ERR_INVALID_ARG;
    if (!aligned16(k_layers[i])) return LOWRAM_ERR_ALIGN;
  }
  if (!aligned16(omega) || !aligned16(basis_out) || !aligned16(workspace)) return LOWRAM_ERR_ALIGN;
  if (evicted(ctx->cfg)) return LOWRAM_ERR_UNSUPPORTED;
  size_t need = 0;
  lowram_status st = lowram_fit_basis_workspace_size(&ctx->cfg, l, &need);
  if (st != LOWRAM_OK) return st;
  if (workspace_bytes < need) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  if (launch_fit_basis(dims_of(ctx->cfg), k_layers, n_layers, omega, l, n_power, basis_out,
                       rope_of(ctx), ctx->status, workspace,
                       static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  return LOWRAM_OK;
}

lowram_status lowram_dense_decode(lowram_ctx* ctx, const void* k_cache, const void* v,
                                  const void* q, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (!ctx || !k_cache || !v || !q || !out || !workspace) return LOWRAM_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v) || !aligned16(q) || !aligned16(out) ||
      !aligned16(workspace))
    return LOWRAM_ERR_ALIGN;
  const Dims dm = dims_of(ctx->cfg);
  if (!dense_supported(dm)) return LOWRAM_ERR_UNSUPPORTED;
  if (workspace_bytes < dense_workspace_bytes(dm)) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  if (launch_dense_decode(dm, k_cache, v, q, out, workspace, ctx->status,
                          static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  return LOWRAM_OK;
}

namespace {
struct SuffixWs {
  size_t out_f32, ml, part, total;
};
SuffixWs suffix_ws(const lowram_config& c, int s_max) {
  const Dims dm = dims_of(c);
  SuffixWs w{};
  size_t o = align_up(decode_ws(c).total);
  w.out_f32 = o; o = align_up(o + (size_t)dm.B * dm.Hq * dm.d * sizeof(float));
  w.ml = o;      o = align_up(o + (size_t)dm.B * dm.Hq * 2 * sizeof(float));
  w.part = o;    o = align_up(o + suffix_workspace_bytes(dm, s_max));
  w.total = o;
  return w;
}
}  // namespace

lowram_status lowram_suffix_workspace_size(const lowram_config* c, int32_t s_max, size_t* bytes) {
  if (!bytes) return LOWRAM_ERR_INVALID_ARG;
  const lowram_status st = lowram_check_config(c);
  if (st != LOWRAM_OK) return st;
  if (s_max < 0) return LOWRAM_ERR_SHAPE;
  if (!dense_supported(dims_of(*c))) return LOWRAM_ERR_UNSUPPORTED;
  *bytes = suffix_ws(*c, s_max).total;
  return LOWRAM_OK;
}

lowram_status lowram_decode_step_suffix(lowram_ctx* ctx, const lowram_cache* cache,
                                        const lowram_layer_params* params, const void* q,
                                        const void* k_suffix, const void* v_suffix,
                                        int32_t s_max, int32_t n_suffix, void* out,
                                        int32_t* sel_out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (!ctx || !q || !out || !workspace) return LOWRAM_ERR_INVALID_ARG;
  if (s_max < 0 || n_suffix < 0 || n_suffix > s_max) return LOWRAM_ERR_SHAPE;
  if (n_suffix > 0 && (!k_suffix || !v_suffix)) return LOWRAM_ERR_INVALID_ARG;
  lowram_status st = check_layer_params(params);
  if (st != LOWRAM_OK) return st;
  if ((st = check_cache(cache, ctx->cfg)) != LOWRAM_OK) return st;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace) ||
      (sel_out && !aligned16(sel_out)) || !aligned16(k_suffix) || !aligned16(v_suffix))
    return LOWRAM_ERR_ALIGN;
  const Dims dm = dims_of(ctx->cfg);
  if (!dense_supported(dm)) return LOWRAM_ERR_UNSUPPORTED;
  const DecodeWs w = decode_ws(ctx->cfg);
  const SuffixWs sw = suffix_ws(ctx->cfg, s_max);
  if (workspace_bytes < sw.total) return LOWRAM_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(ws + w.sel);
  const bool tc = use_tc(ctx->cfg);
  if ((st = select_impl(ctx, cache->landmark, cache->landmark_norm, q, sel, ws, w, s, tc)) !=
      LOWRAM_OK)
    return st;
  float* pre_out = reinterpret_cast<float*>(ws + sw.out_f32);
  float* pre_ml = reinterpret_cast<float*>(ws + sw.ml);
  float* const f32[2] = {pre_out, pre_ml};
  if ((st = attend_impl(ctx, cache, params, q, sel, out, ws, w, s, tc, nullptr, f32)) !=
      LOWRAM_OK)
    return st;
  if (launch_suffix_merge(dm, k_suffix, v_suffix, s_max, n_suffix, q, pre_out, pre_ml, out,
                          ws + sw.part, ctx->status, s) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  return LOWRAM_OK;
}

lowram_status lowram_last_error(lowram_ctx* ctx) {
  if (!ctx) return LOWRAM_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return LOWRAM_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) { cudaGetLastError(); return LOWRAM_ERR_CUDA; }
  int word = 0;
  if (cudaMemcpy(&word, ctx->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(ctx->status, 0, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return LOWRAM_ERR_CUDA;
  }
  if (word & kStatusTimeout) return LOWRAM_ERR_TIMEOUT;
  if (word & kStatusDeviceCheck) return LOWRAM_ERR_DEVICE_CHECK;
  return LOWRAM_OK;
}

const char* lowram_status_string(lowram_status s) {
  switch (s) {
    case LOWRAM_OK: return "ok";
    case LOWRAM_ERR_INVALID_ARG: return "invalid argument";
    case LOWRAM_ERR_SHAPE: return "inconsistent shape";
    case LOWRAM_ERR_ALIGN: return "pointer not 16-byte aligned";
    case LOWRAM_ERR_UNSUPPORTED: return "unsupported size";
    case LOWRAM_ERR_WORKSPACE: return "workspace too small";
    case LOWRAM_ERR_CUDA: return "CUDA error";
    case LOWRAM_ERR_DEVICE_CHECK: return "malformed cache contents detected on the device";
    case LOWRAM_ERR_TIMEOUT: return "a kernel's bounded wait expired";
  }
  return "unknown status";
}

lowram_status lowram_debug_tc_tile(const void* a, const void* b, float* d, int32_t k,
                                   int32_t mode, void* stream) {
  if (!a || !b || !d) return LOWRAM_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(b) || !aligned16(d)) return LOWRAM_ERR_ALIGN;
  if (mode == 0 && (k % 32 != 0 || k < 32 || k > 256)) return LOWRAM_ERR_UNSUPPORTED;
  if ((mode == 1 || mode == 2) && k != 128) return LOWRAM_ERR_UNSUPPORTED;
  if (mode < 0 || mode > 2) return LOWRAM_ERR_INVALID_ARG;
  int* st = nullptr;
  if (cudaMalloc(&st, sizeof(int)) != cudaSuccess) { cudaGetLastError(); return LOWRAM_ERR_CUDA; }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  bool ok = cudaMemsetAsync(st, 0, sizeof(int), s) == cudaSuccess &&
            launch_debug_tc_tile(a, b, d, k, mode, st, s) == cudaSuccess &&
            cudaMemcpyAsync(&word, st, sizeof(int), cudaMemcpyDeviceToHost, s) == cudaSuccess &&
            cudaStreamSynchronize(s) == cudaSuccess;
  cudaFree(st);
  if (!ok) { cudaGetLastError(); return LOWRAM_ERR_CUDA; }
  return word ? LOWRAM_ERR_TIMEOUT : LOWRAM_OK;
}

}  // extern "C"

namespace lowram {
const lowram_config* ctx_config(const lowram_ctx* ctx) { return &ctx->cfg; }
int ctx_device(const lowram_ctx* ctx) { return ctx->device; }
}  // namespace lowram
