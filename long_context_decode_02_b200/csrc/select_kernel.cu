// Kernel (a): landmark scoring and top-k chunk selection for one decode step.
//
// Method: the prefix is cut into chunks whose mean key is a landmark; each decode step
// scores the landmarks with the current query and rebuilds only the top-k chunks
// (LowRAM summary on agihunt.info, paragraph on the key side; cctest "How the method
// works", Selective reconstruction). With GQA a chunk's score is the max over the
// group's query heads of q . L_c; ties go to the lower chunk index.
//
// Structure (HBM-bound: every landmark byte is read once, ~4 FLOP per byte):
//  * Persistent CTAs (one per SM) split the stream of all (batch, KV head) landmark rows
//    into contiguous ranges of stages. A producer warp TMA-loads 64 KB stages (the rows
//    of one (b, h)) into a 3-stage shared-memory ring with the 128-byte swizzle; 256
//    consumer threads each score one landmark row of a stage (packed fp32x2 FMAs against
//    the queries held in shared memory) and write the fp32 score. The swizzle makes the
//    row-per-thread 16-byte reads conflict-free.
//  * The CTA that completes the last stage of a (b, h) (atomic stage counter, no
//    spinning) selects on its consumer warps while its producer keeps streaming:
//    a sorted sample places a threshold, candidates above it are sorted, tau = k-th
//    score, candidates within delta = 1e-3|tau| + 1e-6 max|s| of tau are re-scored in
//    fp64 (exact products, fp64 sums) and ranked by (score desc, index asc). delta is far
//    above the fp32 accumulation error, so the result equals the fp64 selection. When the
//    candidate set cannot be proven to contain the answer, a radix-select path over all
//    scores decides instead. The selection is written in ascending chunk order.
#include <cuda_bf16.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace lowram {
namespace {

using namespace sm100;

constexpr int kConsumers = 256;               // consumer threads (warps 0..7)
constexpr int kSelThreads = kConsumers + 32;  // + producer warp 8
constexpr int kStages = 3;
constexpr int kStageBytes = 65536;
constexpr int kCap = 2048;                    // candidate capacity of the fast selection
constexpr int kSample = 1024;                 // sampled scores placing its threshold
constexpr int kBitmapChunks = 65536;          // chunks the fast path's output bitmap covers
constexpr int kWindowCap = 256;               // fp64 re-scored candidates of the fast path

template <typename T, int D>
struct Geom {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kBoxes = kRowBytes / 128;             // 128-byte column boxes per row
  static constexpr int kBoxCols = 128 / (int)sizeof(T);
  static constexpr int kLps0 = kStageBytes / kRowBytes;
  static constexpr int kLps = kLps0 < kConsumers ? kLps0 : kConsumers;  // rows per stage
  static constexpr int kChunks = kRowBytes / 16;
};

struct SelSmem {  // offsets from the 1024-aligned dynamic base
  uint32_t stages, q, ckey, cid, outs, misc, bar, total;
};
__host__ __device__ inline SelSmem sel_smem(int G, int D) {
  SelSmem L{};
  L.stages = 0;
  L.q = kStages * kStageBytes;
  L.ckey = L.q + (uint32_t)(G * D * 4);
  L.cid = L.ckey + kCap * 4;
  L.outs = L.cid + kCap * 4;            // chunk bitmap of the fast path
  L.misc = L.outs + kBitmapChunks / 8;   // scalars, reduction scratch, window list
  L.bar = L.misc + 3072;
  L.total = L.bar + 128 + 1024;
  return L;
}

struct Misc {
  unsigned hist[256];
  unsigned bc[4];
  float fscr[33];
  int iscr[33];
  int cnt, lo, hi, last;
  float t0, fmax;
  int wl[kWindowCap];
};
static_assert(sizeof(Misc) <= 3072, "Misc scratch");

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

// ---------------------------------------------------------------- selection
// Fallback over all N_c scores: radix select of the k-th largest fp32 score,
// classification against its window, exact fp64 ranking of the window, ascending
// compaction through a flag array.
template <typename T, int D, int G>
__device__ void select_pair_radix(const Grp& g, const SelectArgs& a, int p, Misc* ms) {
  const Dims& dm = a.dm;
  const int Nc = dm.Nc, k = dm.k;
  int32_t* sel = a.sel + (size_t)p * k;
  const float* s = a.scores + (size_t)p * Nc;
  uint8_t* flags = a.flags + (size_t)p * Nc;
  int* cidx = a.cand_idx + (size_t)p * Nc;
  double* cs64 = a.cand_s64 + (size_t)p * Nc;

  float mx = 0.f;
  for (int i = g.tid; i < Nc; i += g.nt) mx = fmaxf(mx, fabsf(__ldcg(s + i)));
  mx = group_max(g, mx, ms->fscr);
  const uint32_t tk = group_kth_largest(
      g, Nc, k, [&](int i) { return f2key(__ldcg(s + i)); }, ms->hist, ms->bc);
  const double tau = (double)key2f(tk);
  const double delta = 1e-3 * fabs(tau) + 1e-6 * (double)mx + 1e-30;
  const double hi = tau + delta, lo = tau - delta;
  if (g.tid == 0) ms->cnt = 0;
  g.sync();
  const int b = p / dm.H, h = p % dm.H;
  const T* qb = (const T*)a.q + ((size_t)b * dm.Hq + (size_t)h * G) * D;
  const T* L = (const T*)a.landmark + (size_t)p * Nc * D;
  int n_in = 0;
  for (int i = g.tid; i < Nc; i += g.nt) {
    const double x = (double)__ldcg(s + i);
    uint8_t f = 0;
    if (x > hi) {
      f = 1;
      ++n_in;
    } else if (x >= lo) {
      f = 2;
      const int slot = atomicAdd(&ms->cnt, 1);
      cidx[slot] = i;
      cs64[slot] = score64<T, D, G>(L + (size_t)i * D, qb);
    }
    flags[i] = f;
  }
  int n_in_total;
  (void)group_exclusive_scan(g, n_in, ms->iscr, &n_in_total);
  const int n_w = ms->cnt;
  const int need = k - n_in_total;
  for (int j = g.tid; j < n_w; j += g.nt) {
    const double sj = cs64[j];
    const int ij = cidx[j];
    int rank = 0;
    for (int m = 0; m < n_w; ++m) {
      const double sm = cs64[m];
      rank += (sm > sj) || (sm == sj && cidx[m] < ij);
    }
    flags[ij] = rank < need ? 1 : 0;
  }
  g.sync();
  int base = 0;
  for (int c0 = 0; c0 < Nc; c0 += g.nt) {
    const int i = c0 + g.tid;
    const int f = (i < Nc && flags[i] == 1) ? 1 : 0;
    int total;
    const int ex = group_exclusive_scan(g, f, ms->iscr, &total);
    if (f && base + ex < k) sel[base + ex] = i;
    base += total;
  }
}

// fp64 score of one landmark row against the group's queries held (exactly, as fp32) in
// shared memory: exact products, one fp64 accumulator per query head.
template <typename T, int D, int G>
__device__ double score64_row(const T* lrow, const float* sQ) {
  constexpr int kV = 16 / (int)sizeof(T);
  double acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = 0.0;
  const uint4* w4 = reinterpret_cast<const uint4*>(lrow);
#pragma unroll 4
  for (int c = 0; c < D / kV; ++c) {
    const uint4 w = w4[c];
    float v[kV];
    if constexpr (sizeof(T) == 2) {
      const float2 a0 = bf2_to_f2(w.x), a1 = bf2_to_f2(w.y), a2 = bf2_to_f2(w.z), a3 = bf2_to_f2(w.w);
      v[0] = a0.x; v[1] = a0.y; v[2] = a1.x; v[3] = a1.y; v[4] = a2.x; v[5] = a2.y; v[6] = a3.x; v[7] = a3.y;
    } else {
      v[0] = __uint_as_float(w.x); v[1] = __uint_as_float(w.y);
      v[2] = __uint_as_float(w.z); v[3] = __uint_as_float(w.w);
    }
#pragma unroll
    for (int e = 0; e < kV; ++e)
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = fma((double)sQ[g * D + c * kV + e], (double)v[e], acc[g]);
  }
  double best = acc[0];
#pragma unroll
  for (int g = 1; g < G; ++g) best = fmax(best, acc[g]);
  return best;
}

// Fast path. Candidates: all scores (N_c <= kCap), or every score at or above a
// threshold t0 = the j-th largest of an evenly spaced sample (radix select). tau = the
// k-th largest candidate (radix select); candidates above tau + delta are in; the window
// |s - tau| <= delta is re-scored in fp64 and ranked by (score desc, index asc); the k
// chosen chunk ids are written ascending through a bitmap scan. Returns false (writing
// nothing) when the candidate set cannot be proven to contain the answer.
template <typename T, int D, int G>
__device__ bool select_pair_fast(const Grp& g, const SelectArgs& a, int p, const float* sQ,
                                 float* ckey, int* cid, uint32_t* bits, Misc* ms) {
  const Dims& dm = a.dm;
  const int Nc = dm.Nc, k = dm.k;
  const int lane = g.tid & 31;
  if (k > kCap / 2 || Nc > kBitmapChunks) return false;
  const float* s = a.scores + (size_t)p * Nc;
  int m;
  float t0 = -INFINITY;
  const bool sampled = Nc > kCap;
  if (!sampled) {
    for (int i = g.tid; i < Nc; i += g.nt) { ckey[i] = __ldcg(s + i); cid[i] = i; }
    m = Nc;
    g.sync();
  } else {
    uint32_t* skey = reinterpret_cast<uint32_t*>(cid);
    for (int i = g.tid; i < kSample; i += g.nt)
      skey[i] = f2key(__ldcg(s + (int)(((long long)i * Nc) / kSample)));
    g.sync();
    int j = (int)((3LL * k * kSample) / (2LL * Nc)) + 16;
    if (j > kSample) j = kSample;
    t0 = key2f(group_kth_largest_aggr(g, kSample, j, [&](int i) { return skey[i]; },
                                      ms->hist, ms->bc));
    if (g.tid == 0) ms->cnt = 0;
    g.sync();
    // every score >= t0 becomes a candidate (warp-aggregated append); each thread issues
    // 8 independent 16-byte loads before filtering them (rows are 16-byte aligned when
    // 4 | N_c; otherwise scalar loads)
    const int n4 = (Nc & 3) == 0 ? Nc / 4 : 0;
    if (n4 == 0) {
      for (int i = g.tid; i < Nc; i += g.nt) {
        const float x = __ldcg(s + i);
        if (x >= t0) {
          const int pos = atomicAdd(&ms->cnt, 1);
          if (pos < kCap) { ckey[pos] = x; cid[pos] = i; }
        }
      }
    }
    const float4* s4 = reinterpret_cast<const float4*>(s);
    for (int base = 0; base < n4; base += 8 * g.nt) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i4 = base + u * g.nt + g.tid;
        v[u] = i4 < n4 ? __ldcg(s4 + i4) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i4 = base + u * g.nt + g.tid;
        const float xs[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * i4 + e;
          const bool keep = i < Nc && xs[e] >= t0;
          const unsigned bal = __ballot_sync(0xffffffffu, keep);
          if (bal == 0) continue;
          int wb = 0;
          if (lane == 0) wb = atomicAdd(&ms->cnt, __popc(bal));
          wb = __shfl_sync(0xffffffffu, wb, 0);
          if (keep) {
            const int pos = wb + __popc(bal & ((1u << lane) - 1u));
            if (pos < kCap) { ckey[pos] = xs[e]; cid[pos] = i; }
          }
        }
      }
    }
    g.sync();
    m = ms->cnt;
    if (m > kCap || m < k) return false;
  }
  const double tau = (double)key2f(group_kth_largest_aggr(
      g, m, k, [&](int i) { return f2key(ckey[i]); }, ms->hist, ms->bc));
  if (g.tid == 0) { ms->cnt = 0; ms->lo = 0; ms->fmax = 0.f; }
  g.sync();
  // |largest candidate| for the window floor
  {
    float mx = 0.f;
    for (int i = g.tid; i < m; i += g.nt) mx = fmaxf(mx, fabsf(ckey[i]));
    mx = warp_max(mx);
    if (lane == 0) atomicMax(reinterpret_cast<int*>(&ms->fmax), __float_as_int(mx));
  }
  for (int i = g.tid; i < kBitmapChunks / 32; i += g.nt) bits[i] = 0u;
  g.sync();
  const double delta = 1e-3 * fabs(tau) + 1e-6 * fmax((double)ms->fmax, fabs(tau)) + 1e-30;
  const double hi = tau + delta, lo = tau - delta;
  if (sampled && (double)t0 > lo) return false;   // the window may reach below the filter
  // classify: clearly in -> bitmap; window -> list (chunk ids in wl, positions in ckey)
  int* wl = reinterpret_cast<int*>(ms->wl);
  for (int i = g.tid; i < m; i += g.nt) {
    const double x = (double)ckey[i];
    if (x > hi) {
      atomicOr(&bits[cid[i] >> 5], 1u << (cid[i] & 31));
      atomicAdd(&ms->lo, 1);
    } else if (x >= lo) {
      const int pos = atomicAdd(&ms->cnt, 1);
      if (pos < kWindowCap) wl[pos] = cid[i];
    }
  }
  g.sync();
  const int n_in = ms->lo, w = ms->cnt, need = k - n_in;
  if (w > kWindowCap) return false;
  const int b = p / dm.H, h = p % dm.H;
  const T* L = (const T*)a.landmark + (size_t)p * Nc * D;
  double* s64 = a.cand_s64 + (size_t)p * Nc;
  for (int i = g.tid; i < w; i += g.nt) s64[i] = score64_row<T, D, G>(L + (size_t)wl[i] * D, sQ);
  (void)b;
  (void)h;
  g.sync();
  for (int i = g.tid; i < w; i += g.nt) {
    const double si = s64[i];
    const int ii = wl[i];
    int rank = 0;
    for (int j2 = 0; j2 < w; ++j2) {
      const double sj = s64[j2];
      rank += (sj > si) || (sj == si && wl[j2] < ii);
    }
    if (rank < need) atomicOr(&bits[ii >> 5], 1u << (ii & 31));
  }
  g.sync();
  // ascending output: exclusive scan of the per-word bit counts
  int32_t* sel = a.sel + (size_t)p * k;
  const int nw = (Nc + 31) / 32;
  int base = 0;
  for (int w0 = 0; w0 < nw; w0 += g.nt) {
    const int wi = w0 + g.tid;
    const uint32_t word = wi < nw ? bits[wi] : 0u;
    int total;
    int pos = base + group_exclusive_scan(g, __popc(word), ms->iscr, &total);
    uint32_t rem = word;
    while (rem) {
      const int bit = __ffs(rem) - 1;
      rem &= rem - 1;
      if (pos < k) sel[pos] = wi * 32 + bit;
      ++pos;
    }
    base += total;
  }
  return true;
}

template <typename T, int D, int G>
__device__ void select_pair(const Grp& g, const SelectArgs& a, int p, const float* sQ,
                            float* ckey, int* cid, uint32_t* bits, Misc* ms) {
  const int Nc = a.dm.Nc, k = a.dm.k;
  if (k >= Nc) {
    int32_t* sel = a.sel + (size_t)p * k;
    for (int i = g.tid; i < Nc; i += g.nt) sel[i] = i;
    return;
  }
  const bool done = select_pair_fast<T, D, G>(g, a, p, sQ, ckey, cid, bits, ms);
  g.sync();
  if (!done) select_pair_radix<T, D, G>(g, a, p, ms);
}

// ---------------------------------------------------------------- scoring
// Score of landmark row r of a swizzled stage.
template <typename T, int D, int G>
__device__ __forceinline__ float score_row(const uint8_t* stage, int r, const float* sQ) {
  using Gm = Geom<T, D>;
  float2 acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < Gm::kChunks; ++c) {
    const int box = c >> 3, cc = c & 7;
    const uint4 w = *reinterpret_cast<const uint4*>(
        stage + box * Gm::kLps * 128 + r * 128 + ((cc ^ (r & 7)) << 4));
    if constexpr (sizeof(T) == 2) {
      // 8 bf16: chunk c holds dims 8c .. 8c+7
      const float2 v0 = bf2_to_f2(w.x), v1 = bf2_to_f2(w.y), v2 = bf2_to_f2(w.z), v3 = bf2_to_f2(w.w);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 q0 = *reinterpret_cast<const float4*>(sQ + g * D + 8 * c);
        const float4 q1 = *reinterpret_cast<const float4*>(sQ + g * D + 8 * c + 4);
        acc[g] = __ffma2_rn(make_float2(q0.x, q0.y), v0, acc[g]);
        acc[g] = __ffma2_rn(make_float2(q0.z, q0.w), v1, acc[g]);
        acc[g] = __ffma2_rn(make_float2(q1.x, q1.y), v2, acc[g]);
        acc[g] = __ffma2_rn(make_float2(q1.z, q1.w), v3, acc[g]);
      }
    } else {
      // 4 fp32: chunk c holds dims 4c .. 4c+3
      const float2 v0 = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
      const float2 v1 = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 q0 = *reinterpret_cast<const float4*>(sQ + g * D + 4 * c);
        acc[g] = __ffma2_rn(make_float2(q0.x, q0.y), v0, acc[g]);
        acc[g] = __ffma2_rn(make_float2(q0.z, q0.w), v1, acc[g]);
      }
    }
  }
  float best = acc[0].x + acc[0].y;
#pragma unroll
  for (int g = 1; g < G; ++g) best = fmaxf(best, acc[g].x + acc[g].y);
  return best;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kSelThreads, 1)
score_select_kernel(const SelectArgs a, const __grid_constant__ CUtensorMap lmap) {
  using Gm = Geom<T, D>;
  const Dims& dm = a.dm;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const SelSmem L = sel_smem(G, D);
  float* sQ = reinterpret_cast<float*>(gbase + L.q);
  float* ckey = reinterpret_cast<float*>(gbase + L.ckey);
  int* cidv = reinterpret_cast<int*>(gbase + L.cid);
  uint32_t* bits = reinterpret_cast<uint32_t*>(gbase + L.outs);
  Misc* ms = reinterpret_cast<Misc*>(gbase + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L.bar + 8 * 2 * kStages);
  auto full = [&](int s) { return base + L.bar + 8u * (uint32_t)s; };
  auto empty = [&](int s) { return base + L.bar + 8u * (uint32_t)(kStages + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Nc = dm.Nc, P = dm.B * dm.H;
  const int upp = (Nc + Gm::kLps - 1) / Gm::kLps;    // stages per (b, h)
  const long long U = (long long)P * upp;
  const int u_begin = (int)(U * blockIdx.x / gridDim.x);
  const int u_end = (int)(U * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kConsumers / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int last_i[kStages];
      for (int s = 0; s < kStages; ++s) last_i[s] = -1;
      for (int u = u_begin, i = 0; u < u_end; ++u, ++i) {
        const int s = i % kStages;
        if (!mbar_wait_bounded(empty(s), ((i / kStages) & 1) ^ 1, abort_flag)) break;
        const int pair = u / upp, st = u % upp;
        const int row = pair * Nc + st * Gm::kLps;
        mbar_arrive_expect_tx(full(s), (uint32_t)(Gm::kBoxes * Gm::kLps * 128));
        for (int bx = 0; bx < Gm::kBoxes; ++bx)
          tma_load_2d(base + L.stages + s * kStageBytes + bx * Gm::kLps * 128, &lmap,
                      bx * Gm::kBoxCols, row, full(s));
        last_i[s] = i;
      }
      if (*abort_flag) {   // loads may still be in flight: let them land before exit
        for (int s = 0; s < kStages; ++s) {
          if (last_i[s] < 0) continue;
          int dummy = 0;
          mbar_wait_bounded(full(s), (last_i[s] / kStages) & 1, (volatile int*)&dummy);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // Every consumer thread runs the same sequence of group barriers whatever its
    // waits return, so a timed-out wait never leaves the others at a barrier.
    const Grp g{(int)threadIdx.x, kConsumers, 1};
    const int tid = threadIdx.x;
    int cur = -1, seg = 0;
    auto finish_segment = [&](int pair, int nst) {
      __threadfence();
      g.sync();
      if (tid == 0) {
        const int old = atomicAdd(a.counters + pair, nst);
        ms->last = (old + nst == upp);
      }
      g.sync();
      if (ms->last) {
        __threadfence();
        select_pair<T, D, G>(g, a, pair, sQ, ckey, cidv, bits, ms);
        g.sync();
        if (tid == 0) a.counters[pair] = 0;
      }
    };
    for (int u = u_begin, i = 0; u < u_end; ++u, ++i) {
      const int pair = u / upp, st = u % upp;
      if (pair != cur) {
        if (cur >= 0) finish_segment(cur, seg);
        cur = pair;
        seg = 0;
        g.sync();
        const int b = pair / dm.H, h = pair % dm.H;
        const T* qb = (const T*)a.q + ((size_t)b * dm.Hq + (size_t)h * G) * D;
        for (int e = tid; e < G * D; e += kConsumers) sQ[e] = ldf(qb, e);
        g.sync();
      }
      const int s = i % kStages;
      mbar_wait_bounded(full(s), (i / kStages) & 1, abort_flag);
      const int c = st * Gm::kLps + tid;
      if (tid < Gm::kLps && c < Nc) {
        const float sc = score_row<T, D, G>(gbase + L.stages + s * kStageBytes, tid, sQ);
        a.scores[(size_t)pair * Nc + c] = sc;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
      ++seg;
    }
    if (cur >= 0) finish_segment(cur, seg);
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) raise_status(a.status, kStatusTimeout);
}

template <typename T, int D, int G>
cudaError_t launch_typed(const SelectArgs& a, int num_sms, cudaStream_t s) {
  using Gm = Geom<T, D>;
  CUtensorMap map;
  if (!make_tensor_map_2d(&map, a.landmark, a.dm.dtype, (uint64_t)D,
                          (uint64_t)a.dm.B * a.dm.H * a.dm.Nc, Gm::kBoxCols, Gm::kLps, 128))
    return cudaErrorInvalidValue;
  const SelSmem L = sel_smem(G, D);
  auto kern = score_select_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L.total);
  if (e != cudaSuccess) return e;
  const long long U = (long long)a.dm.B * a.dm.H * ((a.dm.Nc + Gm::kLps - 1) / Gm::kLps);
  const int grid = (int)(U < num_sms ? U : num_sms);
  kern<<<grid, kSelThreads, L.total, s>>>(a, map);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_by_shape(const SelectArgs& a, int num_sms, cudaStream_t s) {
  const int D = a.dm.d, G = a.dm.G;
#define LR_CASE(DD, GG) \
  if (D == DD && G == GG) return launch_typed<T, DD, GG>(a, num_sms, s);
  LR_CASE(64, 1) LR_CASE(64, 2) LR_CASE(64, 4) LR_CASE(64, 8)
  LR_CASE(128, 1) LR_CASE(128, 2) LR_CASE(128, 4) LR_CASE(128, 8)
#undef LR_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, int num_sms, cudaStream_t s) {
  if (a.dm.dtype == LOWRAM_DTYPE_BF16) return launch_by_shape<__nv_bfloat16>(a, num_sms, s);
  return launch_by_shape<float>(a, num_sms, s);
}

}  // namespace lowram
