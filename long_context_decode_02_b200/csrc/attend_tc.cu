// Kernel (b), tensor-core form: fused reconstruct-and-attend split-K flash-decode on
// tcgen05 / TMEM (bf16 storage, d = 128, F = 256, G = 4, C = 8, r % 32 == 0, r <= 160).
//
// Method (LowRAM summary on agihunt.info, key paragraph and value-amortisation
// paragraph; cctest "How the method works": Low-rank keys, Amortised values, Residuals
// for difficult tokens, Selective reconstruction): rebuild the selected chunks' keys
// from the xKV coefficients and basis, re-apply RoPE, predict their values with the
// per-head MLP plus the stored residuals, and attend over them.
//
// Exact reordering used here: softmax weights sum to one, so
//   sum_t p_t (W2 h_t + b2 + R_t) / sum_t p_t = (W2 (sum_t p_t h_t) + sum_t p_t R_t)/l + b2
// with h_t = act(W1 K~_pre,t + b1): W2 is applied once per query head in the combine
// kernel instead of once per token, removing a third of the tensor work.
//
// Per persistent CTA (one KV head h), per tile of 128 selected tokens (16 chunks of 8),
// 20 warps:
//   warp 0 (TMA)      : B_h once; each tile's 16 chunks' coefficient rows into one of
//                       two coefficient buffers (the next tile's gather under this one).
//   warp 1 (MMA)      : K~_pre as D[tok][d] = coef[tok][r] . B_h[d][r]^T -> TMEM.
//   warp 2 (metadata) : the tile's chunk ids and queries, then its residual list, and
//                       the bulk copies of its chunk-base rotations and bf16 residual rows.
//   warps 3-10 (A)    : K~_pre from TMEM -> bf16 shared memory (the hidden GEMM's
//                       operand); RoPE; logits of the 4 query heads; tile max and
//                       p = 2^(z - m).
//   warp 19 (MMA)     : H^T as D[f][tok] = W1_h[f][d] . K~bf16[tok][d]^T (2 x M = 128),
//                       W1_h held in TMEM.
//   warps 11-18 (B)   : H^T from TMEM (lane = hidden unit f, columns = tokens):
//                       act(h + b1) and Hacc_g[f] += p_g(t) act, a reduction along each
//                       thread's own row; then the tile's residual rows from the staged
//                       row buffer: Racc_g[j] += p_g(t) R_t[j].
//   The tile's (m, l, Hacc, Racc) go to a split-K partial; the combine kernel merges the
//   tiles and applies W2 and b2. Parts A and B run on their own warps at the same time,
//   A one tile ahead; TMEM holds K~ (128 columns), W1_h (128) and H^T (256). Rebuilt keys
//   and values never leave the SM.
// Every wait is bounded (~2 s); on expiry the kernel raises a timeout status, drains its
// own outstanding copies and MMAs (again bounded), frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace lowram {
namespace {

using namespace sm100;

constexpr int kD = 128, kF = 256, kG = 4, kTile = 128, kChunk = 8, kChunksPerTile = 16;
// warp 0 TMA, warp 1 K-MMA issuer + TMEM owner, warp 2 metadata, warps 3..10 epilogue
// part A, warps 11..18 epilogue part B, warp 19 hidden-layer MMA issuer
constexpr int kEpiWarpsA = 8, kEpiWarpsB = 8;
constexpr int kEpiThreadsA = 32 * kEpiWarpsA, kEpiThreadsB = 32 * kEpiWarpsB;
constexpr int kHWarp = 3 + kEpiWarpsA + kEpiWarpsB;
constexpr int kThreads = 32 * (kHWarp + 1);
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128);
constexpr int kPartFloats = 2 * kG + kG * kF + kTcResSlots * kG * kD;

struct TcMaps {
  CUtensorMap coef;   // [B*T][r] bf16, box 64 x 8,  128B swizzle (64-column blocks)
  CUtensorMap coef64; // [B*T][r] bf16, box 32 x 8,   64B swizzle (a last 32-column block)
  CUtensorMap basis;  // [H*d][r] bf16, box 32 x 128, 64B swizzle
};

// One slot of the metadata ring (filled by the metadata warp up to kMetaSlots tiles
// ahead; read by the TMA warp and the epilogue; released after the epilogue's part B).
struct TileMeta {
  int cid[kChunksPerTile];  // chunk id of each slot of the tile; -1 past the selection
  int nres;                 // residual rows of the tile
  int item;                 // b * n_tiles + tile; -1: this CTA has no more tiles
  int nstaged;              // residual entries 0 .. nstaged-1 are in the tile's row buffer
  int pad;
  uint32_t res[kTile];      // (row of res_val) << 8 | token row in the tile (255 = skip)
  uint4 q[64];              // the tile's G = 4 query rows, bf16 [4][128]
};
static_assert(sizeof(TileMeta) == 1616, "TileMeta layout");
constexpr int kMetaSlots = 4;
// bf16 residual rows of a tile are copied into one of two row buffers by the metadata
// warp (bulk copies of each chunk's contiguous span); entries past kResCap (a tile with
// more than 48 of its 128 tokens residual) are read from global memory
constexpr int kResCap = 48;
constexpr int kResBufs = 2;

constexpr int kRotSlots = 2;   // chunk-base rotations, one slot per tile in flight
// float2 stride of a chunk's 64 rotations: padded by 2 so the four chunks one warp reads
// fall in different shared-memory banks
constexpr int kRotStride = kD / 2 + 2;

constexpr uint32_t kBarBytes = 320;   // mbarriers, the TMEM address and the abort word

struct Layout {
  uint32_t basis, coef, kbf, p, p2, q, b1, zx, red, rot, roff, meta, rbuf, bar, total;
};
__host__ __device__ constexpr uint32_t align_up(uint32_t x, uint32_t a) {
  return (x + a - 1) / a * a;
}
__host__ __device__ inline Layout make_layout(int r) {
  Layout L{};
  const uint32_t kb = (uint32_t)r / 32;
  L.basis = 0;
  L.coef = align_up(L.basis + kb * 8192, 1024);   // two coefficient tile buffers
  L.kbf = align_up(L.coef + 2 * kb * 8192, 1024);  // K~ bf16 [128 tok][128 d], one buffer
  L.p = L.kbf + 32768;          // [2][128][4] fp32
  L.p2 = L.p + 4096;            // [2][64 token pairs][4][2] fp32: P by token pairs
  L.q = L.p2 + 4096;            // [4][64][2] fp32: (q_x, q_y) of each rotary pair
  L.b1 = L.q + 2048;            // [256] fp32
  L.zx = L.b1 + 1024;           // [128][4] fp32: the second pair half's partial logits
  L.red = L.zx + 2048;          // 512 B of reduction scratch
  L.rot = L.red + 512;          // [kRotSlots][16 chunks][kRotStride] float2 (cos, sin)
  L.roff = L.rot + kRotSlots * kChunksPerTile * kRotStride * 8;  // [64 pairs][8] float2
  L.meta = L.roff + (kD / 2) * kChunk * 8;  // kMetaSlots x TileMeta
  L.rbuf = align_up(L.meta + kMetaSlots * (uint32_t)sizeof(TileMeta), 128);  // residual rows
  L.bar = L.rbuf + kResBufs * kResCap * kD * 2;   // barriers + TMEM holder
  L.total = L.bar + kBarBytes + 1024;  // + alignment slack of the dynamic base
  return L;
}

// barrier slots (8 bytes each) inside L.bar
enum {
  BAR_W = 0, BAR_W1T, BAR_COEF_FULL0, BAR_COEF_FULL1, BAR_COEF_EMPTY0, BAR_COEF_EMPTY1,
  BAR_KT_FULL, BAR_KT_EMPTY, BAR_KBF_FULL, BAR_KBF_EMPTY, BAR_H_FULL, BAR_H_EMPTY, BAR_DRAIN, BAR_DRAIN_H,
  BAR_P_FULL0, BAR_P_FULL1, BAR_P_EMPTY0, BAR_P_EMPTY1,
  BAR_ROT_FULL0, BAR_ROT_EMPTY0 = BAR_ROT_FULL0 + kRotSlots,
  BAR_META_FULL0 = BAR_ROT_EMPTY0 + kRotSlots, BAR_META_EMPTY0 = BAR_META_FULL0 + kMetaSlots,
  BAR_RES_FULL0 = BAR_META_EMPTY0 + kMetaSlots,   // a slot's residual list (and rows) landed
  BAR_RBUF_EMPTY0 = BAR_RES_FULL0 + kMetaSlots,   // part B is done with a residual row buffer
  BAR_COUNT = BAR_RBUF_EMPTY0 + kResBufs
};
static_assert(BAR_COUNT * 8 + 8 <= kBarBytes, "barrier area");

template <int ACT>
__device__ __forceinline__ float act_fast(float x) {
  if (ACT == LOWRAM_ACT_SILU) {
    const float hx = 0.5f * x;
    return fmaf(hx, tanh_approx(hx), hx);   // x * sigmoid(x) = x/2 (1 + tanh(x/2))
  }
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

// Polls *flag until it is non-zero, with acquire semantics (bounded: 2 s, or *abort set;
// on giving up sets *abort and returns 0).
// Reduces four values per lane over the warp in one reduce-scatter (6 shuffles instead
// of 4 x 5): every lane of lane group lane >> 3 gets the reduction of value lane >> 3.
template <typename Op>
__device__ __forceinline__ float warp_reduce4_scatter(const float (&v)[4], int lane, Op op) {
  const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0;
  const float u0 = op(b4 ? v[2] : v[0], __shfl_xor_sync(0xffffffffu, b4 ? v[0] : v[2], 16));
  const float u1 = op(b4 ? v[3] : v[1], __shfl_xor_sync(0xffffffffu, b4 ? v[1] : v[3], 16));
  float w = op(b3 ? u1 : u0, __shfl_xor_sync(0xffffffffu, b3 ? u0 : u1, 8));
  w = op(w, __shfl_xor_sync(0xffffffffu, w, 4));
  w = op(w, __shfl_xor_sync(0xffffffffu, w, 2));
  w = op(w, __shfl_xor_sync(0xffffffffu, w, 1));
  return w;
}

// Polls *word (acquire) until it has bit `bit`; returns the word (0 after giving up: 2 s,
// or the abort flag, which is then set).
__device__ uint32_t wait_bit_acquire(const int* word, int bit, volatile int* abort) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(word) : "memory");
    if ((v >> bit) & 1u) return v;
    if (*abort) return 0;
    if (global_timer_ns() - t0 > 2000000000ull) break;
    __nanosleep(256);
  }
  *abort = 1;
  return 0;
}

// DBG (test only): also store the rebuilt rows (a.dbg_k, a.dbg_h, a.dbg_v) where the
// epilogue holds them; the product instantiation has DBG = false and stores nothing.
template <int ACT, bool DBG>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const AttendArgs a, const __grid_constant__ TcMaps maps) {
  const Dims& dm = a.dm;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = align_up(raw, 1024);
  uint8_t* gbase = smem_raw + (base - raw);
  const Layout L = make_layout(dm.r);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // KV heads interleaved over the grid, so CTAs that start early (beside a still running
  // selection kernel) serve every head; each head's tiles are taken from its counter
  const int h = blockIdx.x % dm.H;
  const int n_items = dm.B * a.n_tiles;
  const int kb_r = dm.r / 32;
  const int ksteps_r = dm.r / 16;
  const int n128 = dm.r / 64;            // 64-column coefficient blocks (128B swizzle)
  const bool has64 = (dm.r & 63) != 0;   // and a last 32-column block (64B swizzle)

  auto bar = [&](int i) { return base + L.bar + 8u * (uint32_t)i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + L.bar + 8 * BAR_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L.bar + 8 * BAR_COUNT + 4);
  float* sP = reinterpret_cast<float*>(gbase + L.p);
  float* sQ = reinterpret_cast<float*>(gbase + L.q);
  float* sP2 = reinterpret_cast<float*>(gbase + L.p2);
  float* sB1 = reinterpret_cast<float*>(gbase + L.b1);
  float* sZx = reinterpret_cast<float*>(gbase + L.zx);
  float* sRed = reinterpret_cast<float*>(gbase + L.red);  // [4 quadrants][4 g] x 2, ml[2][4][2]
  TileMeta* meta = reinterpret_cast<TileMeta*>(gbase + L.meta);
  float2* sRot = reinterpret_cast<float2*>(gbase + L.rot);
  float2* sRoff = reinterpret_cast<float2*>(gbase + L.roff);

  auto item_of = [&](int it, int& b, int& tile) {
    b = it / a.n_tiles;
    tile = it % a.n_tiles;
  };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(BAR_W), 1);
    mbar_init(bar(BAR_W1T), kEpiWarpsA + kEpiWarpsB);
    for (int c = 0; c < 2; ++c) {
      mbar_init(bar(BAR_COEF_FULL0 + c), 1);
      mbar_init(bar(BAR_COEF_EMPTY0 + c), 1);
    }
    mbar_init(bar(BAR_KT_FULL), 1);
    mbar_init(bar(BAR_KT_EMPTY), kEpiWarpsA);
    mbar_init(bar(BAR_KBF_FULL), kEpiWarpsA);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_P_FULL0 + i), 1);
      mbar_init(bar(BAR_P_EMPTY0 + i), kEpiWarpsB);
    }
    mbar_init(bar(BAR_KBF_EMPTY), 1);
    for (int i = 0; i < kRotSlots; ++i) {
      mbar_init(bar(BAR_ROT_FULL0 + i), 1);
      mbar_init(bar(BAR_ROT_EMPTY0 + i), kEpiWarpsA);
    }
    mbar_init(bar(BAR_H_FULL), 1);
    mbar_init(bar(BAR_DRAIN_H), 1);
    mbar_init(bar(BAR_H_EMPTY), kEpiWarpsB);
    mbar_init(bar(BAR_DRAIN), 1);
    for (int i = 0; i < kMetaSlots; ++i) {
      mbar_init(bar(BAR_META_FULL0 + i), 1);
      mbar_init(bar(BAR_META_EMPTY0 + i), kEpiWarpsB);
      mbar_init(bar(BAR_RES_FULL0 + i), 1);
    }
    for (int i = 0; i < kResBufs; ++i) mbar_init(bar(BAR_RBUF_EMPTY0 + i), kEpiWarpsB);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // the combine kernel may start on SMs this kernel leaves; it waits for this grid's
  // completion before it reads the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int32_t* sel_all = a.sel;
  // W1_h into Tensor Memory as the hidden-layer GEMM's A operand: row f = 128 hf + lane
  // of half hf in lane `lane`, columns 128 + 64 hf + (0..63) holding bf16 pairs along d.
  // Each epilogue warp (quadrant of trow, half hf, d-half dh) writes 32 columns from one
  // batch of eight 16-byte loads per thread.
  auto w1_to_tmem = [&](int hf, int dh, int trow, uint32_t lane_addr) {
    const uint4* wrow = reinterpret_cast<const uint4*>(
        (const __nv_bfloat16*)a.w1 + ((size_t)h * kF + 128 * hf + trow) * kD + 64 * dh);
    uint32_t v[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 x = __ldg(wrow + j);
      v[4 * j] = x.x;
      v[4 * j + 1] = x.y;
      v[4 * j + 2] = x.z;
      v[4 * j + 3] = x.w;
    }
    const uint32_t col = tmem + lane_addr + 128u + (uint32_t)(64 * hf + 32 * dh);
    tmem_st_x16(col, v);
    tmem_st_x16(col + 16, v + 16);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar(BAR_W1T));
  };
  if (warp == 0) {
    // ------------------------------------------------------------ TMA warp
    // The basis once; then per tile the coefficient rows of its 16 chunks (chunk ids from
    // the tile's metadata slot), TMA-gathered into one of two tile buffers, so the next
    // tile's gather overlaps this tile's GEMM.
    int last0 = -1, last1 = -1;   // last tile loaded into each buffer (for the drain)
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(BAR_W), (uint32_t)(kb_r * 8192));
      for (int kb = 0; kb < kb_r; ++kb)
        tma_load_2d(base + L.basis + kb * 8192, &maps.basis, kb * 32, h * kD, bar(BAR_W));
    }
    for (int i = 0;; ++i) {
      const int slot = i % kMetaSlots;
      int got = 0, it = -1;
      if (lane == 0) {
        got = mbar_wait_bounded(bar(BAR_META_FULL0 + slot), (i / kMetaSlots) & 1, abort_flag);
        it = got ? meta[slot].item : -1;
        if (it >= 0)
          got = mbar_wait_bounded(bar(BAR_COEF_EMPTY0 + (i & 1)), ((i >> 1) & 1) ^ 1, abort_flag);
      }
      it = __shfl_sync(0xffffffffu, it, 0);
      if (!__shfl_sync(0xffffffffu, got, 0) || it < 0) break;
      int b, tile;
      item_of(it, b, tile);
      const int cid = lane < kChunksPerTile ? meta[slot].cid[lane] : -1;
      // each chunk: r/64 boxes of 64 columns (128B swizzle) and, when 64 does not divide
      // r, one box of the last 32 columns (64B swizzle): 3 boxes per chunk at r = 160
      const uint32_t cbuf = base + L.coef + (uint32_t)((i & 1) * kb_r * 8192);
      const uint32_t cfull = bar(BAR_COEF_FULL0 + (i & 1));
      if (lane == 0) mbar_arrive_expect_tx(cfull, (uint32_t)(kChunksPerTile * kb_r * 512));
      __syncwarp();
      if (lane < kChunksPerTile) {
        const int row = b * dm.T + (cid < 0 ? 0 : cid) * kChunk;
        for (int c2 = 0; c2 < n128; ++c2)
          tma_load_2d(cbuf + c2 * 16384 + lane * 1024, &maps.coef, c2 * 64, row, cfull);
        if (has64)
          tma_load_2d(cbuf + n128 * 16384 + lane * 512, &maps.coef64, n128 * 64, row, cfull);
      }
      if (i & 1) last1 = i; else last0 = i;
    }
    // drain: loads still in flight (only possible after an abort) must land before exit
    if (lane == 0 && *abort_flag) {
      for (int c = 0; c < 2; ++c) {
        const int li = c ? last1 : last0;
        if (li < 0) continue;
        int dummy = 0;
        mbar_wait_bounded(bar(BAR_COEF_FULL0 + c), (uint32_t)((li >> 1) & 1),
                          (volatile int*)&dummy);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ metadata warp
    // Per tile: chunk ids, the residual rows of its chunks (CSR spans, every index
    // bounds-checked), its queries, and the rotation of each chunk's base position,
    // up to kMetaSlots (kRotSlots for rotations) tiles ahead of the epilogue.
    // The four dependent global reads of a tile (its item from the head's counter, its
    // chunk ids, their CSR spans, the residual rows) are software-pipelined over four
    // tiles: one pass of the loop issues the counter take of tile j + 3, the spans of
    // j + 1 and the residual rows of j, posts tile j, then issues the chunk ids of j + 2,
    // so a tile costs about one memory round trip instead of four.
    const int32_t* ptr_all = a.chunk_ptr;
    const int32_t* ridx_all = a.res_idx;
    // tiles come from this head's counter (lane 0 takes, the warp learns it later); the
    // first tile of the c-th CTA of the head is tile c, so the counter starts after them
    const int ctas_h = ((int)gridDim.x - h + dm.H - 1) / dm.H;   // CTAs serving head h
    auto take_raw = [&]() -> int {
      return lane == 0 ? ctas_h + atomicAdd(a.item_ctr + h, 1) : 0;
    };
    // chunk ids of item `it` (issued, not waited for); -1 past the selection
    auto load_cid = [&](int it) -> int {
      int b, tile;
      item_of(it, b, tile);
      int cid = -1;
      if (lane < kChunksPerTile) {
        const int gs = tile * kChunksPerTile + lane;
        if (gs < dm.k) cid = __ldcg(sel_all + ((size_t)b * dm.H + h) * dm.k + gs);
      }
      return cid;
    };
    // when the selection kernel may still be running: wait until item it's pair is
    // published (acquire on the head's readiness word); false after a timeout (the abort
    // flag is then set). Bits once seen stay set for the launch, so every pair (b < 64)
    // a read has shown published is remembered and not read again.
    uint64_t seen_ready = 0;
    auto pair_ready = [&](int it) -> bool {
      if (!a.wait_ready) return true;
      int b, tile;
      item_of(it, b, tile);
      if (b < 64 && ((seen_ready >> b) & 1ull)) return true;
      uint32_t w = 1;
      if (lane == 0) w = wait_bit_acquire(a.ready + ready_word(dm, b, h), b & 31, abort_flag);
      w = __shfl_sync(0xffffffffu, w, 0);
      if (w == 0) return false;
      if (b < 64) seen_ready |= (uint64_t)w << (b & 32);
      return true;
    };
    // an id outside [-1, Nc) is reported and dropped (the chunk is skipped)
    auto sanitize = [&](int cid) -> int {
      if (lane < kChunksPerTile && (cid >= dm.Nc || cid < -1)) {
        raise_status(a.status, kStatusDeviceCheck);
        return -1;
      }
      return cid;
    };
    // CSR span reads of item it's chunk cid (issued, validated one stage later)
    auto load_span = [&](int it, int cid, int& e0, int& e1) {
      e0 = 0;
      e1 = 0;
      if (it < n_items && lane < kChunksPerTile && cid >= 0) {
        int b, tile;
        item_of(it, b, tile);
        const int32_t* ptr = ptr_all + (size_t)(b * dm.H + h) * (dm.Nc + 1);
        e0 = ptr[cid];
        e1 = ptr[cid + 1];
      }
    };
    int rot_issued = -1;   // last tile whose rotations were requested (for the drain)
    int res_issued = -1;   // last tile whose residual rows were requested (for the drain)
    // the queries of item it (issued, written into the slot when it is posted)
    auto load_q = [&](int it, uint4& qa, uint4& qb) {
      qa = make_uint4(0u, 0u, 0u, 0u);
      qb = qa;
      if (it < n_items) {
        int b, tile;
        item_of(it, b, tile);
        const uint4* qsrc = reinterpret_cast<const uint4*>(
            (const __nv_bfloat16*)a.q + ((size_t)b * dm.Hq + (size_t)h * kG) * kD);
        qa = qsrc[lane];
        qb = qsrc[lane + 32];
      }
    };
    // prologue: the CTA's own first tile and two tiles from the counter; chunk ids and
    // queries of tile 0, chunk ids of tile 1, spans of tile 0
    int tk1 = take_raw(), tk2 = take_raw();
    int it0 = (int)blockIdx.x / dm.H;
    int cid0 = -1, cid1 = -1;
    if (it0 < n_items && pair_ready(it0)) cid0 = load_cid(it0);
    uint4 qa0, qb0;
    load_q(it0, qa0, qb0);
    int it1 = __shfl_sync(0xffffffffu, tk1, 0);
    int it2 = __shfl_sync(0xffffffffu, tk2, 0);
    if (it1 < n_items && pair_ready(it1)) cid1 = load_cid(it1);
    cid0 = sanitize(cid0);
    int e0r, e1r;
    load_span(it0, cid0, e0r, e1r);
    for (int i = 0;; ++i) {
      const int it = it0;
      const int slot = i % kMetaSlots;
      int got = 0;
      if (lane == 0)
        got = mbar_wait_bounded(bar(BAR_META_EMPTY0 + slot), ((i / kMetaSlots) & 1) ^ 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      TileMeta* M = meta + slot;
      if (it >= n_items) {   // no more tiles: post the end marker
        if (lane == 0) {
          M->item = -1;
          mbar_arrive(bar(BAR_META_FULL0 + slot));
        }
        break;
      }
      int b, tile;
      item_of(it, b, tile);
      const int p = b * dm.H + h;
      const int cid = cid0;
      // first half of the slot: chunk ids, queries, item. The coefficient gather, the K~
      // GEMM and part A need nothing else, so they start before the residual reads below.
      if (lane < kChunksPerTile) M->cid[lane] = cid;
      M->q[lane] = qa0;
      M->q[lane + 32] = qb0;
      if (lane == 0) M->item = it;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_META_FULL0 + slot));
      // chunk-base rotations (cos, sin)(C cid theta_i) of the tile's chunks: one 512-byte
      // row of the context's table per chunk, copied by the TMA engine (row 0 for a slot
      // past the selection)
      {
        const int rs = i % kRotSlots;
        int rgot = 0;
        if (lane == 0)
          rgot = mbar_wait_bounded(bar(BAR_ROT_EMPTY0 + rs), ((i / kRotSlots) & 1) ^ 1, abort_flag);
        if (!__shfl_sync(0xffffffffu, rgot, 0)) break;
        const uint32_t rfull = bar(BAR_ROT_FULL0 + rs);
        if (lane == 0) mbar_arrive_expect_tx(rfull, (uint32_t)(kChunksPerTile * (kD / 2) * 8));
        __syncwarp();
        if (lane < kChunksPerTile) {
          // the chunk's original position (eviction), bounds-checked
          const int cpos = cid < 0 ? 0 : chunk_position(dm, a.chunk_pos, b, cid, a.status);
          bulk_load(smem_u32(sRot + (rs * kChunksPerTile + lane) * kRotStride),
                    a.rope.chunk32 + (size_t)cpos * (kD / 2), (kD / 2) * 8, rfull);
        }
        rot_issued = i;
      }
      // issue: the take of tile i + 3, the residual rows of tile i (its spans arrived in
      // the previous pass), the queries and spans of tile i + 1, the chunk ids of tile i + 2
      const int tk3 = take_raw();
      int e0 = 0, n = 0;
      if (lane < kChunksPerTile && cid >= 0) {
        if (e0r < 0 || e1r < e0r || e1r > dm.n_res || e1r - e0r > kChunk) {
          raise_status(a.status, kStatusDeviceCheck);
        } else {
          e0 = e0r;
          n = e1r - e0r;
        }
      }
      const int32_t* ridx = ridx_all + (size_t)p * dm.n_res + e0;
      int t[kChunk];
#pragma unroll
      for (int j = 0; j < kChunk; ++j) t[j] = j < n ? ridx[j] : 0;
      load_q(it1, qa0, qb0);
      cid1 = sanitize(cid1);
      load_span(it1, cid1, e0r, e1r);
      int cid2 = -1;
      if (it2 < n_items && pair_ready(it2)) cid2 = load_cid(it2);
      // second half of the slot: the tile's residual list for part B and, for bf16 rows,
      // the rows themselves: each chunk's span (contiguous in res_val) is bulk-copied into
      // the tile's row buffer once part B is done with that buffer's previous tile
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int off = incl - n;
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      const bool stage = dm.res_int4 == 0;
      const int rb = i % kResBufs;
      if (stage) {
        int eg = 0;
        if (lane == 0)
          eg = mbar_wait_bounded(bar(BAR_RBUF_EMPTY0 + rb), ((i / kResBufs) & 1) ^ 1, abort_flag);
        if (!__shfl_sync(0xffffffffu, eg, 0)) break;
      }
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        if (j < n) {
          const int tt = t[j] - cid * kChunk;
          const bool good = tt >= 0 && tt < kChunk;
          if (!good) raise_status(a.status, kStatusDeviceCheck);
          M->res[off + j] = ((uint32_t)(e0 + j) << 8) | (good ? (uint32_t)(lane * kChunk + tt) : 255u);
        }
      }
      const int nst = stage ? min(total, kResCap) : 0;
      if (lane == 0) {
        M->nres = total;
        M->nstaged = nst;
      }
      __syncwarp();
      const uint32_t rfull = bar(BAR_RES_FULL0 + slot);
      if (lane == 0) mbar_arrive_expect_tx(rfull, (uint32_t)(nst * kD * 2));
      __syncwarp();
      const int ncp = stage ? max(0, min(n, kResCap - off)) : 0;   // this chunk's staged rows
      if (ncp > 0)
        bulk_load(smem_u32(gbase + L.rbuf) + (uint32_t)((rb * kResCap + off) * kD * 2),
                  (const __nv_bfloat16*)a.res_val + ((size_t)p * dm.n_res + e0) * kD,
                  (uint32_t)(ncp * kD * 2), rfull);
      res_issued = i;
      // advance the pipeline
      it0 = it1;
      it1 = it2;
      it2 = __shfl_sync(0xffffffffu, tk3, 0);
      cid0 = cid1;
      cid1 = cid2;
    }
    // drain: rotation and residual-row copies still in flight (only possible after an
    // abort) land first
    if (lane == 0 && *abort_flag) {
      for (int t = rot_issued - kRotSlots + 1; t <= rot_issued; ++t) {
        if (t < 0) continue;
        int dummy = 0;
        mbar_wait_bounded(bar(BAR_ROT_FULL0 + t % kRotSlots), (uint32_t)((t / kRotSlots) & 1),
                          (volatile int*)&dummy);
      }
      for (int t = res_issued - kResBufs + 1; t <= res_issued; ++t) {
        if (t < 0) continue;
        int dummy = 0;
        mbar_wait_bounded(bar(BAR_RES_FULL0 + t % kMetaSlots), (uint32_t)((t / kMetaSlots) & 1),
                          (volatile int*)&dummy);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar(BAR_W), 0, abort_flag);
      const uint32_t sb = base + L.basis, sc0 = base + L.coef;
      auto issue_k = [&](int i) -> bool {
        const int c = i & 1;   // coefficient buffer
        if (!mbar_wait_bounded(bar(BAR_COEF_FULL0 + c), (i >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait_bounded(bar(BAR_KT_EMPTY), (i & 1) ^ 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d_t = tmem;   // K~ (one buffer, columns 0..127)
        const uint32_t sc = sc0 + (uint32_t)(c * kb_r * 8192);
        for (int s = 0; s < ksteps_r; ++s) {
          const uint32_t off = (uint32_t)((s >> 1) * 8192 + (s & 1) * 32);   // basis
          const uint64_t adesc =
              s < 4 * n128
                  ? smem_desc_kmajor(sc + (uint32_t)((s >> 2) * 16384 + (s & 3) * 32), 1024,
                                     kSwizzle128B)
                  : smem_desc_kmajor(sc + (uint32_t)(n128 * 16384 + (s & 1) * 32), 512,
                                     kSwizzle64B);
          mma_bf16(d_t, adesc, smem_desc_kmajor(sb + off, 512, kSwizzle64B), kIdesc, s > 0);
        }
        mma_commit(bar(BAR_KT_FULL));
        mma_commit(bar(BAR_COEF_EMPTY0 + c));
        return true;
      };
      // whether tile i exists, from its metadata slot (read before the slot can recycle)
      auto exists = [&](int i) -> bool {
        const int slot = i % kMetaSlots;
        if (!mbar_wait_bounded(bar(BAR_META_FULL0 + slot), (i / kMetaSlots) & 1, abort_flag))
          return false;
        return meta[slot].item >= 0;
      };
      // the K~ GEMMs run ahead on their own: the hidden-layer GEMMs have their own issuer
      for (int i = 0; ok && exists(i); ++i) ok = issue_k(i);
      // drain every MMA this thread issued before TMEM is released
      mma_commit(bar(BAR_DRAIN));
      int dummy = 0;
      mbar_wait_bounded(bar(BAR_DRAIN), 0, (volatile int*)&dummy);
    }
  } else if (warp == kHWarp) {
    // ------------------------------------------------------------ hidden-layer MMA issuer
    if (lane == 0) {
      // W1_h is the A operand, in Tensor Memory (columns 128 + 64 hf ..), written there by
      // the part-A warps at the start
      bool ok = mbar_wait_bounded(bar(BAR_W1T), 0, abort_flag);
      const uint32_t skb = base + L.kbf;
      for (int i = 0; ok; ++i) {
        const int slot = i % kMetaSlots;
        if (!mbar_wait_bounded(bar(BAR_META_FULL0 + slot), (i / kMetaSlots) & 1, abort_flag) ||
            meta[slot].item < 0)
          break;
        if (!mbar_wait_bounded(bar(BAR_KBF_FULL), i & 1, abort_flag)) break;
        if (!mbar_wait_bounded(bar(BAR_H_EMPTY), (i & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t d_t = tmem + 256u + (uint32_t)hf * 128u;
          for (int s = 0; s < 8; ++s) {
            const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
            mma_bf16_ta(d_t, tmem + 128u + (uint32_t)(hf * 64 + 8 * s),
                        smem_desc_kmajor(skb + off, 1024, kSwizzle128B), kIdesc, s > 0);
          }
        }
        mma_commit(bar(BAR_H_FULL));
        mma_commit(bar(BAR_KBF_EMPTY));
      }
      mma_commit(bar(BAR_DRAIN_H));
      int dummy = 0;
      mbar_wait_bounded(bar(BAR_DRAIN_H), 0, (volatile int*)&dummy);
    }
  } else if (warp < 3 + kEpiWarpsA) {
    // ------------------------------------------------------------ epilogue, part A
    // 8 warps, two per TMEM lane quadrant: pair half ha of the tile's tokens' K~ rows;
    // RoPE, logits, K~ in bf16 for the hidden-layer GEMM, softmax weights P. Part B runs
    // concurrently on its own 8 warps; P passes between them through a 2-slot ring.
    const int ea = warp - 3;             // 0..7
    const int qd = warp & 3;             // TMEM lane quadrant this warp may access
    const int ha = ea >> 2;              // pair half
    const int et = threadIdx.x - 96;     // 0..255
    const int trow = 32 * qd + lane;     // token row
    const uint32_t lane_addr = (uint32_t)(32 * qd) << 16;
    const float zscale = 1.4426950408889634f * rsqrtf((float)kD);
    float* s_ml = sRed + 64;  // [2][4][2]
    w1_to_tmem(ha, 0, trow, lane_addr);
    // in-chunk offsets: sRoff[pair * 8 + j] = (cos, sin)(j theta_pair), j < 8
    for (int i = et; i < (kD / 2) * kChunk; i += kEpiThreadsA)
      sRoff[i] = a.rope.lo32[(i & (kChunk - 1)) * (kD / 2) + (i >> 3)];
    // A failed (timed-out) wait never changes the sequence of named barriers: the
    // thread carries on with `good` false so every barrier is still reached. Returns false
    // when the tile does not exist (the end marker) or a wait gave up, decided by one vote.
    auto part_a = [&](int i) -> bool {
      const int u = i & 1;
      const int slot = i % kMetaSlots;
      const TileMeta* M = meta + slot;
      bool good = mbar_wait_bounded(bar(BAR_META_FULL0 + slot), (i / kMetaSlots) & 1, abort_flag);
      // the vote is also the barrier after which the previous readers of sQ / sZx are done
      if (named_bar_red_or(1, kEpiThreadsA, !good || M->item < 0)) {
        if (!good) *abort_flag = 1;
        return false;
      }
      const bool valid = M->cid[trow >> 3] >= 0;
      float* dbg_krow = nullptr;   // this token's K~_rot row (DBG only)
      if constexpr (DBG) {
        int b, tile;
        item_of(M->item, b, tile);
        if (valid)
          dbg_krow = a.dbg_k + (((size_t)b * dm.H + h) * dm.k * kChunk + (size_t)tile * kTile + trow) * kD;
      }
      {   // sQ[g][i][w] = q_g[i + 64 w]: each rotary pair's two query components adjacent
        const uint32_t w = reinterpret_cast<const uint32_t*>(M->q)[et];
        const float2 f = bf2_to_f2(w);
        const int g = et >> 6, d0 = 2 * (et & 63), hw = d0 >> 6, i0 = d0 & 63;
        sQ[g * kD + 2 * i0 + hw] = f.x;
        sQ[g * kD + 2 * i0 + 2 + hw] = f.y;
      }
      good = mbar_wait_bounded(bar(BAR_KT_FULL), i & 1, abort_flag) && good;
      const int rs = i % kRotSlots;
      good = mbar_wait_bounded(bar(BAR_ROT_FULL0 + rs), (i / kRotSlots) & 1, abort_flag) && good;
      named_bar_sync(1, kEpiThreadsA);  // sQ ready
      // K~_pre in bf16 goes to shared memory (single buffer, 128B-swizzled K-major
      // [tok][d]) once the previous tile's hidden-layer MMA has released it
      good = mbar_wait_bounded(bar(BAR_KBF_EMPTY), (i & 1) ^ 1, abort_flag) && good;
      tc_fence_after();
      const uint32_t skb = base + L.kbf;
      const float4* rbase4 = reinterpret_cast<const float4*>(
          sRot + (rs * kChunksPerTile + (trow >> 3)) * kRotStride);
      float2 z2[kG];
#pragma unroll
      for (int g = 0; g < kG; ++g) z2[g] = make_float2(0.f, 0.f);
#pragma unroll 1
      for (int sb = 0; sb < 2; ++sb) {
        // pairs p0 .. p0 + 15 of this thread's token: K~ columns p0.. and 64 + p0..
        const int p0 = 32 * ha + 16 * sb;
        float x[16], y[16];
        const uint32_t tcol = tmem + lane_addr + (uint32_t)p0;
        tmem_ld_x16(tcol, x);
        tmem_ld_x16(tcol + 64, y);
        tmem_wait_ld();
        if (sb == 1) {   // both halves of this thread's K~ columns are in registers
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_KT_EMPTY));
        }
        // RoPE on pairs (p0 + e, 64 + p0 + e): the chunk-base rotation (from the ring)
        // times the in-chunk offset (table) by angle addition; partial logits accumulate as
        // (x, y) pairs with packed fp32x2 FMAs, the queries of 4 pairs in one 16-byte load
        const float4* rb4 = rbase4 + p0 / 2;
        const float2* ro = sRoff + p0 * kChunk + (trow & 7);
#pragma unroll
        for (int e4 = 0; e4 < 16; e4 += 4) {
          const float4 b01 = rb4[e4 / 2], b23 = rb4[e4 / 2 + 1];
          const float2 bs[4] = {make_float2(b01.x, b01.y), make_float2(b01.z, b01.w),
                                make_float2(b23.x, b23.y), make_float2(b23.z, b23.w)};
          float2 rot[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int e = e4 + w;
            const float2 cs = rope_combine(bs[w], ro[e * kChunk]);
            rot[w] = make_float2(x[e] * cs.x - y[e] * cs.y, x[e] * cs.y + y[e] * cs.x);
            if constexpr (DBG) {
              if (dbg_krow) {
                dbg_krow[p0 + e] = rot[w].x;
                dbg_krow[kD / 2 + p0 + e] = rot[w].y;
              }
            }
          }
          const int pi = p0 + e4;
#pragma unroll
          for (int g = 0; g < kG; ++g) {
            const float4 qa = *reinterpret_cast<const float4*>(sQ + g * kD + 2 * pi);
            const float4 qb = *reinterpret_cast<const float4*>(sQ + g * kD + 2 * pi + 4);
            z2[g] = __ffma2_rn(make_float2(qa.x, qa.y), rot[0], z2[g]);
            z2[g] = __ffma2_rn(make_float2(qa.z, qa.w), rot[1], z2[g]);
            z2[g] = __ffma2_rn(make_float2(qb.x, qb.y), rot[2], z2[g]);
            z2[g] = __ffma2_rn(make_float2(qb.z, qb.w), rot[3], z2[g]);
          }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ch = (p0 >> 3) + cc;   // 16-byte chunk of the 64-dim block
          st_shared_v4(skb + sw128_offset(trow, ch),
                       pack_bf16x2(x[8 * cc + 0], x[8 * cc + 1]), pack_bf16x2(x[8 * cc + 2], x[8 * cc + 3]),
                       pack_bf16x2(x[8 * cc + 4], x[8 * cc + 5]), pack_bf16x2(x[8 * cc + 6], x[8 * cc + 7]));
          st_shared_v4(skb + 16384 + sw128_offset(trow, ch),
                       pack_bf16x2(y[8 * cc + 0], y[8 * cc + 1]), pack_bf16x2(y[8 * cc + 2], y[8 * cc + 3]),
                       pack_bf16x2(y[8 * cc + 4], y[8 * cc + 5]), pack_bf16x2(y[8 * cc + 6], y[8 * cc + 7]));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_ROT_EMPTY0 + rs));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_KBF_FULL));
      float z[kG];
#pragma unroll
      for (int g = 0; g < kG; ++g) z[g] = z2[g].x + z2[g].y;

      if (ha == 1) *reinterpret_cast<float4*>(sZx + 4 * trow) = make_float4(z[0], z[1], z[2], z[3]);
      named_bar_sync(1, kEpiThreadsA);
      if (ha == 0) {
        const float4 o = *reinterpret_cast<const float4*>(sZx + 4 * trow);
        z[0] = valid ? (z[0] + o.x) * zscale : -INFINITY;
        z[1] = valid ? (z[1] + o.y) * zscale : -INFINITY;
        z[2] = valid ? (z[2] + o.z) * zscale : -INFINITY;
        z[3] = valid ? (z[3] + o.w) * zscale : -INFINITY;
        {   // per-quadrant maxima of the four heads
          const float m = warp_reduce4_scatter(z, lane, [](float x, float y) { return fmaxf(x, y); });
          if ((lane & 7) == 0) sRed[qd * 4 + (lane >> 3)] = m;
        }
        // P slot u is free once part B has finished with tile i - 2
        int pe = 1;
        if (lane == 0) pe = mbar_wait_bounded(bar(BAR_P_EMPTY0 + u), ((i >> 1) & 1) ^ 1, abort_flag);
        good = __shfl_sync(0xffffffffu, pe, 0) && good;
        named_bar_sync(2, 128);
        float m[kG], pv[kG];
#pragma unroll
        for (int g = 0; g < kG; ++g) {
          m[g] = fmaxf(fmaxf(sRed[g], sRed[4 + g]), fmaxf(sRed[8 + g], sRed[12 + g]));
          pv[g] = valid ? ex2_approx(z[g] - m[g]) : 0.f;
        }
        *reinterpret_cast<float4*>(sP + u * 512 + 4 * trow) = make_float4(pv[0], pv[1], pv[2], pv[3]);
        {   // sP2[u][t / 2][g][t % 2]: the weights of tokens 2m and 2m + 1 side by side
          float po[kG];
#pragma unroll
          for (int g = 0; g < kG; ++g) po[g] = __shfl_down_sync(0xffffffffu, pv[g], 1);
          if ((lane & 1) == 0) {
            float4* d2 = reinterpret_cast<float4*>(sP2 + u * 512 + 4 * trow);
            d2[0] = make_float4(pv[0], po[0], pv[1], po[1]);
            d2[1] = make_float4(pv[2], po[2], pv[3], po[3]);
          }
        }
        {   // per-quadrant sums of the four heads' weights
          const float l = warp_reduce4_scatter(pv, lane, [](float x, float y) { return x + y; });
          if ((lane & 7) == 0) sRed[16 + qd * 4 + (lane >> 3)] = l;
        }
        named_bar_sync(2, 128);
        if (ea == 0 && lane < kG) {
          const int g = lane;
          s_ml[u * 8 + g * 2 + 0] = m[g];
          s_ml[u * 8 + g * 2 + 1] = sRed[16 + g] + sRed[20 + g] + sRed[24 + g] + sRed[28 + g];
        }
      }
      named_bar_sync(1, kEpiThreadsA);  // P and (m, l) of tile i written
      if (et == 0) mbar_arrive(bar(BAR_P_FULL0 + u));
      if (!good) *abort_flag = 1;
      return true;
    };
    // after a failed wait every later wait returns at once and the vote ends the loop
    for (int i = 0; part_a(i); ++i) {
    }
  } else {
    // ------------------------------------------------------------ epilogue, part B
    // 8 warps, two per TMEM lane quadrant: hidden half hf of H^T (lane = hidden unit f,
    // columns = the tile's 128 tokens): act(h + b1) and Hacc_g[f] += p_g(t) act, a
    // reduction along each thread's own TMEM row; and the residual rows of the tile.
    const int eb = warp - 3 - kEpiWarpsA;   // 0..7
    const int qd = warp & 3;
    const int hf = eb >> 2;
    const int etb = threadIdx.x - 96 - kEpiThreadsA;   // 0..255
    const int trow = 32 * qd + lane;
    const uint32_t lane_addr = (uint32_t)(32 * qd) << 16;
    const __nv_bfloat16* rval_all = (const __nv_bfloat16*)a.res_val;
    const float* s_ml = sRed + 64;
    w1_to_tmem(hf, 1, trow, lane_addr);
    for (int i = etb; i < kF; i += kEpiThreadsB)
      sB1[i] = __bfloat162float(((const __nv_bfloat16*)a.b1)[(size_t)h * kF + i]);
    named_bar_sync(3, kEpiThreadsB);
    auto part_b = [&](int i) -> bool {
      const int u = i & 1;
      const int slot = i % kMetaSlots;
      const TileMeta* M = meta + slot;
      bool good = mbar_wait_bounded(bar(BAR_META_FULL0 + slot), (i / kMetaSlots) & 1, abort_flag);
      if (named_bar_red_or(3, kEpiThreadsB, !good || M->item < 0)) {
        if (!good) *abort_flag = 1;
        return false;
      }
      int b, tile;
      item_of(M->item, b, tile);
      const int p = b * dm.H + h;
      float* part = a.part + ((size_t)p * a.n_tiles + tile) * kPartFloats;
      // first debug row of this tile (DBG only); a row is stored only if its chunk exists
      const size_t dbg_row0 = ((size_t)p * dm.k * kChunk + (size_t)tile * kTile);
      // residual rows of the tile: thread = column j, rows split between the two halves
      const int j = trow;
      const __nv_bfloat16* rbase = rval_all + (size_t)p * dm.n_res * kD + j;
      const bool q4 = dm.res_int4 != 0;   // int4 rows are read from global memory
      good = mbar_wait_bounded(bar(BAR_P_FULL0 + u), (i >> 1) & 1, abort_flag) && good;
      good = mbar_wait_bounded(bar(BAR_H_FULL), i & 1, abort_flag) && good;
      tc_fence_after();
      const int f = 128 * hf + trow;
      const float bias = sB1[f];
      float2 hacc01 = make_float2(0.f, 0.f), hacc23 = make_float2(0.f, 0.f);
      float2 acc2[kG];   // per head: (even tokens, odd tokens)
#pragma unroll
      for (int g = 0; g < kG; ++g) acc2[g] = make_float2(0.f, 0.f);
      const float4* P4 = reinterpret_cast<const float4*>(sP + u * 512);
      const float4* P2 = reinterpret_cast<const float4*>(sP2 + u * 512);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float hv[32];
        tmem_ld_x32(tmem + lane_addr + 256u + (uint32_t)(hf * 128 + 32 * c), hv);
        tmem_wait_ld();
        if (c == 3) {   // all of H^T is in registers: the next tile's hidden-layer GEMM may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_H_EMPTY));
        }
        if (ACT == LOWRAM_ACT_SILU) {
          // two tokens per step: hx = (h + b1)/2, silu = hx + hx tanh(hx)
          const float2 half2 = make_float2(0.5f, 0.5f);
          const float2 hb2 = make_float2(0.5f * bias, 0.5f * bias);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 hx = __ffma2_rn(half2, make_float2(hv[e], hv[e + 1]), hb2);
            const float2 av = __ffma2_rn(hx, make_float2(tanh_approx(hx.x), tanh_approx(hx.y)), hx);
            if constexpr (DBG) {
              const int t0 = 32 * c + e;
              if (M->cid[t0 >> 3] >= 0) a.dbg_h[(dbg_row0 + t0) * kF + f] = av.x;
              if (M->cid[(t0 + 1) >> 3] >= 0) a.dbg_h[(dbg_row0 + t0 + 1) * kF + f] = av.y;
            }
            const float4 pa = P2[32 * c + e], pb = P2[32 * c + e + 1];   // tokens (e, e + 1)
            acc2[0] = __ffma2_rn(make_float2(pa.x, pa.y), av, acc2[0]);
            acc2[1] = __ffma2_rn(make_float2(pa.z, pa.w), av, acc2[1]);
            acc2[2] = __ffma2_rn(make_float2(pb.x, pb.y), av, acc2[2]);
            acc2[3] = __ffma2_rn(make_float2(pb.z, pb.w), av, acc2[3]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float av = act_fast<ACT>(hv[e] + bias);
            if constexpr (DBG) {
              if (M->cid[(32 * c + e) >> 3] >= 0) a.dbg_h[(dbg_row0 + 32 * c + e) * kF + f] = av;
            }
            const float4 pv = P4[32 * c + e];
            hacc01 = __ffma2_rn(make_float2(pv.x, pv.y), make_float2(av, av), hacc01);
            hacc23 = __ffma2_rn(make_float2(pv.z, pv.w), make_float2(av, av), hacc23);
          }
        }
      }
      if (ACT == LOWRAM_ACT_SILU) {
        hacc01 = make_float2(acc2[0].x + acc2[0].y, acc2[1].x + acc2[1].y);
        hacc23 = make_float2(acc2[2].x + acc2[2].y, acc2[3].x + acc2[3].y);
      }
      part[2 * kG + 0 * kF + f] = hacc01.x;
      part[2 * kG + 1 * kF + f] = hacc01.y;
      part[2 * kG + 2 * kF + f] = hacc23.x;
      part[2 * kG + 3 * kF + f] = hacc23.y;

      // V~ = MLP + R on the residual rows: the list and (bf16) the rows, copied into the
      // tile's row buffer by the metadata warp, are waited for only now
      good = mbar_wait_bounded(bar(BAR_RES_FULL0 + slot), (i / kMetaSlots) & 1, abort_flag) && good;
      const int nres = good ? M->nres : 0;
      const int nst = good ? M->nstaged : 0;
      const __nv_bfloat16* rstage = reinterpret_cast<const __nv_bfloat16*>(gbase + L.rbuf) +
                                    (size_t)(i % kResBufs) * kResCap * kD + j;
      float racc[kG] = {0.f, 0.f, 0.f, 0.f};
      // this half's entries ei = hf, hf + 2, ... in batches of four, whose loads are all
      // issued before the sums (accumulated in entry order)
      for (int e4 = hf; e4 < nres; e4 += 8) {
        uint32_t ent[4];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) ent[k2] = e4 + 2 * k2 < nres ? M->res[e4 + 2 * k2] : 255u;
        float r[4];
        float4 pv[4];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          const int ei = e4 + 2 * k2;
          const uint32_t row = ent[k2] & 255u;
          r[k2] = 0.f;
          pv[k2] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (row != 255u) {
            r[k2] = q4 ? int4_residual((const uint8_t*)a.res_val, (const __half*)a.res_scale, dm,
                                       (size_t)p * dm.n_res + (ent[k2] >> 8), j)
                       : __bfloat162float(ei < nst ? rstage[(size_t)ei * kD]
                                                   : rbase[(size_t)(ent[k2] >> 8) * kD]);
            pv[k2] = P4[row];
          }
        }
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          const uint32_t row = ent[k2] & 255u;
          if (row == 255u) continue;
          if constexpr (DBG) a.dbg_v[(dbg_row0 + row) * kD + j] = r[k2];
          racc[0] = fmaf(pv[k2].x, r[k2], racc[0]);
          racc[1] = fmaf(pv[k2].y, r[k2], racc[1]);
          racc[2] = fmaf(pv[k2].z, r[k2], racc[2]);
          racc[3] = fmaf(pv[k2].w, r[k2], racc[3]);
        }
      }
      if (!q4) {   // the row buffer may take tile i + kResBufs
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_RBUF_EMPTY0 + i % kResBufs));
      }
      float* pr = part + 2 * kG + kG * kF + (size_t)hf * kG * kD;
#pragma unroll
      for (int g = 0; g < kG; ++g) pr[g * kD + j] = racc[g];
      if (eb == 0 && lane < 2 * kG) part[lane] = s_ml[u * 8 + lane];
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(BAR_P_EMPTY0 + u));
        mbar_arrive(bar(BAR_META_EMPTY0 + slot));
      }
      if (!good) *abort_flag = 1;
      return true;
    };
    for (int i = 0; part_b(i); ++i) {
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) raise_status(a.status, kStatusTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // when launched as a programmatic dependent of the selection kernel, finish only after
  // it has: the kernels that follow in the stream then find it complete as well
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// --------------------------------------------------------------------- debug tile
// d[m][n] = sum_k a[m][k] b[n][k]. mode 0: both operands TMA-loaded with the 64B swizzle
// exactly as coef (8-row boxes) and basis (128-row boxes) in the decode kernel; mode 1:
// a TMA-loaded with the 128B swizzle like W1, b written by threads with the 128B swizzle
// like K~bf16 (K = 128); mode 2: a (128 x 128) written by threads into TMEM as bf16
// pairs and read by the MMA from there, b (16 x 128) written by threads with the 128B
// swizzle, D = 128 x 16.
__global__ void __launch_bounds__(128, 1)
debug_tc_tile_kernel(const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mb,
                     const __nv_bfloat16* asrc, const __nv_bfloat16* bsrc, float* d, int K,
                     int mode, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = align_up(raw, 1024);
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sa = base, sb = base + 65536;
  const uint32_t barf = base + 131072, bard = barf + 8;
  uint32_t* holder = reinterpret_cast<uint32_t*>(gbase + 131072 + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + 131072 + 20);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(barf, 1);
    mbar_init(bard, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(holder), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  const int kb32 = K / 32;
  if (mode == 1) {
    // b by threads: row n = threadIdx.x, 128B-swizzled K-major, two 64-wide K blocks
    const int n = threadIdx.x;
    for (int c = 0; c < 16; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(bsrc + (size_t)n * 128 + 8 * c);
      st_shared_v4(sb + (c >> 3) * 16384 + sw128_offset(n, c & 7), v.x, v.y, v.z, v.w);
    }
    fence_proxy_async_smem();
  }
  if (mode == 2) {
    // a row m = threadIdx.x -> TMEM lane m, columns 0..63 (two bf16 per column)
    const uint32_t* arow = reinterpret_cast<const uint32_t*>(asrc + (size_t)threadIdx.x * 128);
    for (int c = 0; c < 4; ++c) {
      uint32_t v[16];
      for (int j = 0; j < 16; ++j) v[j] = arow[16 * c + j];
      tmem_st_x16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(16 * c), v);
    }
    tmem_wait_st();
    // b rows 0..15, 128B-swizzled K-major, two 64-wide K blocks of 16 rows
    if (threadIdx.x < 16) {
      const int n = threadIdx.x;
      for (int c = 0; c < 16; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(bsrc + (size_t)n * 128 + 8 * c);
        st_shared_v4(sb + (c >> 3) * 2048 + sw128_offset(n, c & 7), v.x, v.y, v.z, v.w);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    if (mode == 2) {
      tc_fence_after();
      for (int s = 0; s < 8; ++s)
        mma_bf16_ta(tmem + 64u, tmem + (uint32_t)(8 * s),
                    smem_desc_kmajor(sb + (uint32_t)((s >> 2) * 2048 + (s & 3) * 32), 1024,
                                     kSwizzle128B),
                    idesc_bf16_f32(128, 16), s > 0);
    } else if (mode == 0) {
      mbar_arrive_expect_tx(barf, (uint32_t)(2 * kb32 * 8192));
      for (int kb = 0; kb < kb32; ++kb) {
        for (int c = 0; c < 16; ++c) tma_load_2d(sa + kb * 8192 + c * 512, &ma, kb * 32, c * 8, barf);
        tma_load_2d(sb + kb * 8192, &mb, kb * 32, 0, barf);
      }
    } else {
      mbar_arrive_expect_tx(barf, 2u * 16384u);
      for (int kb = 0; kb < 2; ++kb) tma_load_2d(sa + kb * 16384, &ma, kb * 64, 0, barf);
    }
    if (mode != 2) ok = mbar_wait_bounded(barf, 0, abort_flag);
    if (ok && mode != 2) {
      tc_fence_after();
      if (mode == 0) {
        for (int s = 0; s < K / 16; ++s) {
          const uint32_t off = (uint32_t)((s >> 1) * 8192 + (s & 1) * 32);
          mma_bf16(tmem, smem_desc_kmajor(sa + off, 512, kSwizzle64B),
                   smem_desc_kmajor(sb + off, 512, kSwizzle64B), kIdesc, s > 0);
        }
      } else {
        for (int s = 0; s < 8; ++s) {
          const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
          mma_bf16(tmem, smem_desc_kmajor(sa + off, 1024, kSwizzle128B),
                   smem_desc_kmajor(sb + off, 1024, kSwizzle128B), kIdesc, s > 0);
        }
      }
    }
    mma_commit(bard);
    if (!mbar_wait_bounded(bard, 0, abort_flag)) ok = false;
    if (!ok) raise_status(status, kStatusTimeout);
  }
  __syncthreads();
  tc_fence_after();
  if (!*abort_flag && mode == 2) {
    float v[32];
    tmem_ld_x32(tmem + ((uint32_t)(32 * warp) << 16) + 64u, v);
    tmem_wait_ld();
    for (int e = 0; e < 16; ++e) d[(size_t)threadIdx.x * 128 + e] = v[e];
  } else if (!*abort_flag) {
    const int m = threadIdx.x;  // warp w reads lanes 32w..32w+31
    for (int c = 0; c < 4; ++c) {
      float v[32];
      tmem_ld_x32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(32 * c), v);
      tmem_wait_ld();
      for (int e = 0; e < 32; ++e) d[(size_t)m * 128 + 32 * c + e] = v[e];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// --------------------------------------------------------------------- host helpers
}  // namespace

bool attend_tc_supported(const Dims& dm) {
  return dm.dtype == LOWRAM_DTYPE_BF16 && dm.d == kD && dm.F == kF && dm.G == kG &&
         dm.C == kChunk && dm.r % 32 == 0 && dm.r >= 32 && dm.r <= 160 &&
         (dm.act == LOWRAM_ACT_SILU || dm.act == LOWRAM_ACT_GELU_ERF) &&
         (dm.k * kChunk + kTile - 1) / kTile <= 64;
}

size_t attend_tc_part_floats(const Dims& dm, int n_tiles) {
  return (size_t)dm.B * dm.H * n_tiles * kPartFloats;
}

cudaError_t launch_attend_tc(const AttendArgs& a, int num_sms, cudaStream_t s) {
  const Dims& dm = a.dm;
  TcMaps maps;
  if (!make_tensor_map_2d(&maps.coef, a.coef, LOWRAM_DTYPE_BF16, dm.r, (uint64_t)dm.B * dm.T, 64, 8, 128) ||
      !make_tensor_map_2d(&maps.coef64, a.coef, LOWRAM_DTYPE_BF16, dm.r, (uint64_t)dm.B * dm.T, 32, 8, 64) ||
      !make_tensor_map_2d(&maps.basis, a.basis, LOWRAM_DTYPE_BF16, dm.r, (uint64_t)dm.H * kD, 32, 128, 64))
    return cudaErrorInvalidValue;
  const Layout L = make_layout(dm.r);
  const int n_items = dm.B * a.n_tiles;
  int cph = num_sms / dm.H;
  if (cph < 1) cph = 1;
  if (cph > n_items) cph = n_items;
  cudaError_t e;
  const bool dbg = a.dbg_k != nullptr;
  auto kern = dm.act == LOWRAM_ACT_SILU
                  ? (dbg ? attend_tc_kernel<LOWRAM_ACT_SILU, true> : attend_tc_kernel<LOWRAM_ACT_SILU, false>)
                  : (dbg ? attend_tc_kernel<LOWRAM_ACT_GELU_ERF, true>
                         : attend_tc_kernel<LOWRAM_ACT_GELU_ERF, false>);
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)L.total)) != cudaSuccess) return e;
  // after the selection kernel: a programmatic dependent launch, so CTAs start on SMs
  // the selection kernel has left and overlap its last selections
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(dm.H * cph);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.wait_ready ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, a, maps);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Test only: v[row][j] += b2_h[j] + sum_f W2_h[j][f] act[row][f] for every rebuilt row
// (one CTA per row, thread j), in fp32 from the stored bf16 weights.
__global__ void __launch_bounds__(kD) debug_values_kernel(const AttendArgs a) {
  const Dims& dm = a.dm;
  const size_t row = blockIdx.x;
  const int h = (int)((row / ((size_t)dm.k * kChunk)) % dm.H);
  const int j = threadIdx.x;
  const float* hr = a.dbg_h + row * kF;
  const __nv_bfloat16* w2 = (const __nv_bfloat16*)a.w2 + ((size_t)h * kD + j) * kF;
  float acc = __bfloat162float(((const __nv_bfloat16*)a.b2)[(size_t)h * kD + j]);
  for (int f = 0; f < kF; ++f) acc = fmaf(__bfloat162float(w2[f]), hr[f], acc);
  a.dbg_v[row * kD + j] += acc;
}

cudaError_t launch_debug_values(const AttendArgs& a, cudaStream_t s) {
  const size_t rows = (size_t)a.dm.B * a.dm.H * a.dm.k * kChunk;
  if (rows == 0) return cudaSuccess;
  debug_values_kernel<<<(unsigned)rows, kD, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_debug_tc_tile(const void* a, const void* b, float* d, int k, int mode,
                                 int* status, cudaStream_t s) {
  CUtensorMap ma, mb;
  if (mode == 2) {
    memset(&ma, 0, sizeof(ma));
    mb = ma;
  } else if (mode == 0) {
    if (!make_tensor_map_2d(&ma, a, LOWRAM_DTYPE_BF16, (uint64_t)k, 128, 32, 8, 64) ||
        !make_tensor_map_2d(&mb, b, LOWRAM_DTYPE_BF16, (uint64_t)k, 128, 32, 128, 64))
      return cudaErrorInvalidValue;
  } else {
    if (!make_tensor_map_2d(&ma, a, LOWRAM_DTYPE_BF16, 128, 128, 64, 128, 128))
      return cudaErrorInvalidValue;
    mb = ma;
  }
  const int smem = 131072 + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(debug_tc_tile_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  debug_tc_tile_kernel<<<1, 128, smem, s>>>(ma, mb, (const __nv_bfloat16*)a,
                                            (const __nv_bfloat16*)b, d, k, mode, status);
  return cudaGetLastError();
}

}  // namespace lowram
