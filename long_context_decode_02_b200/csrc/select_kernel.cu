// Kernel (a): landmark scoring and top-k chunk selection for one decode step.
//
// Method: the prefix is cut into chunks whose mean key is a landmark; each decode step
// scores the landmarks with the current query and rebuilds only the top-k chunks
// (LowRAM summary on agihunt.info, paragraph on the key side; cctest "How the method
// works", Selective reconstruction). With GQA a chunk's score is the max over the
// group's query heads of q . L_c; ties go to the lower chunk index.
//
// Structure (HBM-bound: every landmark byte is read once, ~4 FLOP per byte):
//  * Persistent CTAs (one per SM) take 64 KB stages (up to 256 landmark rows of one
//    (b, h)) from a global work counter in (b, h)-major order, so the load balances
//    itself and the (b, h) pairs are completed one after another while the stream runs.
//    A producer warp TMA-loads each stage into a 3-stage shared-memory ring (128-byte
//    swizzle) and stages the pair's queries in fp32 beside it; 256 consumer threads
//    score the rows (packed fp32x2 FMAs; bf16 rows by lane pairs, each lane one half of
//    the dims of two rows, so each query load serves two rows) and write fp32 scores.
//  * Scores live in a context-owned buffer that holds a sentinel bit pattern between
//    launches (0xFFFFFFFF, a NaN that fp32 arithmetic never produces), so a written score
//    is its own completion flag: no counters or memory fences on the streaming path.
//    Three selection warps per CTA take (b, h) pairs in order from a global counter,
//    wait until the work counter has handed out all of the pair's stages and every score
//    has landed, select, set the pair's readiness bit and put the sentinel back.
//    Selections are spread over the CTAs and overlap the stream; a selection group only
//    waits for stages held by running CTAs, and every wait is bounded. Pairs whose
//    scoring ends in the last wave of stages are selected by the whole CTA once its
//    stream is done.
//  * Selection: the 16-bit key prefix of the j-th largest of 1024 evenly spaced scores
//    gives a threshold t0; every score >= t0 is a candidate; three radix passes find the
//    24-bit prefix bucket [tau_lo, tau_hi] holding the k-th largest candidate.
//    Candidates above tau_hi + delta are in; those in [tau_lo - delta, tau_hi + delta]
//    are re-scored in fp64 (exact products, fp64 sums) and ranked by (score desc, index
//    asc). delta is twice a rigorous bound on the fp32 score error: an fp32 dot product of
//    D terms accumulated with fused multiply-adds is within gamma_D * sum|q_i L_i| <=
//    gamma_D * |q|_2 |L|_2 of the exact value (gamma_n = n u / (1 - n u), u = 2^-24), with
//    |L|_2 bounded by the cache's per-pair landmark norm. So the result equals the
//    selection made in fp64, and the window usually holds exactly the rows still
//    needed, which then need no re-scoring. When the candidate set cannot be proven to
//    hold the answer, a radix select over all scores decides instead. The chunk ids are
//    written in ascending order.
#include <cuda_bf16.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace lowram {
namespace {

using namespace sm100;

constexpr int kConsumers = 256;               // consumer threads (warps 0..7)
constexpr int kSelectors = 96;                // selection threads (warps 9..11)
// stages per CTA that count as the last wave: more for long pairs, whose selections
// beside the stream are slow (measured: 10 best at N_c 16384, 16 at N_c 32768)
constexpr int kLateWaves = 10;
constexpr int kLateWavesLong = 16;
constexpr int kLongPair = 16384;              // N_c above which kLateWavesLong applies
constexpr int kJoinBar = 3;                   // named barrier of the joint selection group
constexpr int kSelThreads = kConsumers + 32 + kSelectors;  // + producer warp 8
constexpr int kStages = 3;
constexpr int kStageBytes = 65536;
constexpr int kSample = 1024;                 // sampled scores placing the threshold t0
constexpr int kBitmapChunks = 65536;          // chunks the fast path's output bitmap covers
constexpr int kWindowCap = 256;               // fp64 re-scored candidates of the fast path
constexpr int kSmemLimit = 232448;            // opt-in shared memory per block

// Candidate capacity of the fast selection: smaller when the per-stage queries are large.
__host__ __device__ constexpr int cand_cap(int G, int D) { return G * D <= 512 ? 2048 : 1280; }

template <typename T, int D>
struct Geom {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kBoxes = kRowBytes / 128;             // 128-byte column boxes per row
  static constexpr int kBoxCols = 128 / (int)sizeof(T);
  static constexpr int kLps0 = kStageBytes / kRowBytes;
  static constexpr int kLps = kLps0 < kConsumers ? kLps0 : kConsumers;  // rows per stage
  static constexpr int kChunks = kRowBytes / 16;
};


struct Misc {
  unsigned hist[512];   // two radix histograms
  unsigned bc[4];
  unsigned kr[2];       // smallest and largest key of a radix search
  float fscr[33];
  int iscr[33];
  int cnt, n_in, nwin;
  float fmax;           // largest landmark norm among the candidates
  int req;              // the selection group's current request
  int carry;            // a claimed pair handed from the selection warps to the whole group
  int wl[kWindowCap];
};

struct SelSmem {  // offsets from the 1024-aligned dynamic base
  uint32_t stages, q, ckey, cid, outs, misc, hdr, bar, total;
};
__host__ __device__ inline SelSmem sel_smem(int G, int D) {
  SelSmem L{};
  const int cap = cand_cap(G, D);
  L.stages = 0;
  L.q = kStages * kStageBytes;                          // fp32 queries per stage
  L.ckey = L.q + (uint32_t)(kStages * G * D * 4);
  L.cid = L.ckey + cap * 4;
  L.outs = L.cid + cap * 4;                              // chunk bitmap of the fast path
  L.misc = L.outs + kBitmapChunks / 8;
  L.hdr = L.misc + (uint32_t)((sizeof(Misc) + 15) & ~(size_t)15);   // stage units
  L.bar = L.hdr + 64;       // full[], empty[], abort word
  L.total = L.bar + 64 + 1024;
  return L;
}
static_assert(kStages * 4 <= 64 && 2 * kStages * 8 + 4 <= 64, "stage units and barriers");

constexpr uint32_t kScoreEmpty = 0xFFFFFFFFu;   // sentinel of an unwritten score

__device__ __forceinline__ void or_release(int* p, uint32_t bits) {
  asm volatile("red.release.gpu.global.or.b32 [%0], %1;" ::"l"(p), "r"(bits) : "memory");
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint4 ld_relaxed4(const uint32_t* p) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p) : "memory");
  return v;
}

// Polls *p until it reaches target (bounded: 2 s, or *abort set; on giving up sets *abort).
__device__ bool wait_counter_ge(const int* p, int target, volatile int* abort) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if ((int)ld_relaxed(reinterpret_cast<const uint32_t*>(p)) >= target) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > 2000000000ull) break;
    __nanosleep(500);
  }
  *abort = 1;
  return false;
}

// Waits until none of the n scores at sp holds the sentinel (this thread's share of the
// group; bounded like wait_counter_ge). Returns false on giving up.
__device__ bool wait_scores(const Grp& g, const uint32_t* sp, int n, volatile int* abort) {
  const uint64_t t0 = global_timer_ns();
  const bool vec = (reinterpret_cast<uintptr_t>(sp) & 15) == 0;
  for (int i = 4 * g.tid; i < n; i += 4 * g.nt) {
    for (;;) {
      bool done;
      if (vec && i + 4 <= n) {
        const uint4 v = ld_relaxed4(sp + i);
        done = v.x != kScoreEmpty && v.y != kScoreEmpty && v.z != kScoreEmpty && v.w != kScoreEmpty;
      } else {
        done = true;
        for (int e = i; e < n && e < i + 4; ++e) done = done && ld_relaxed(sp + e) != kScoreEmpty;
      }
      if (done) break;
      if (*abort) return false;
      if (global_timer_ns() - t0 > 2000000000ull) { *abort = 1; return false; }
      __nanosleep(200);
    }
  }
  return true;
}

// Puts the sentinel back into n scores (this thread's share).
__device__ void clear_scores(const Grp& g, uint32_t* sp, int n) {
  const bool vec = (reinterpret_cast<uintptr_t>(sp) & 15) == 0;
  for (int i = 4 * g.tid; i < n; i += 4 * g.nt) {
    if (vec && i + 4 <= n)
      *reinterpret_cast<uint4*>(sp + i) = make_uint4(kScoreEmpty, kScoreEmpty, kScoreEmpty, kScoreEmpty);
    else
      for (int e = i; e < n && e < i + 4; ++e) sp[e] = kScoreEmpty;
  }
}

// Loads the kN words su[idx[j]] for the bits j of want, polling until none holds the
// sentinel; returns false if the wait gave up (2 s since t0, or *abort set).
template <int kN>
__device__ bool poll_words(const uint32_t* su, const int (&idx)[kN], uint32_t want,
                           uint32_t (&v)[kN], volatile int* abort, uint64_t t0) {
  while (want) {
#pragma unroll
    for (int j = 0; j < kN; ++j)
      if ((want >> j) & 1u) v[j] = ld_relaxed(su + idx[j]);
#pragma unroll
    for (int j = 0; j < kN; ++j)
      if (((want >> j) & 1u) && v[j] != kScoreEmpty) want &= ~(1u << j);
    if (!want) break;
    if (*abort) return false;
    if (global_timer_ns() - t0 > 2000000000ull) { *abort = 1; return false; }
    __nanosleep(200);
  }
  return true;
}

// The same for kN 16-byte groups su[4 idx[j] .. 4 idx[j] + 3].
template <int kN>
__device__ bool poll_vec4(const uint32_t* su, const int (&idx)[kN], uint32_t want,
                          uint4 (&v)[kN], volatile int* abort, uint64_t t0) {
  while (want) {
#pragma unroll
    for (int j = 0; j < kN; ++j)
      if ((want >> j) & 1u) v[j] = ld_relaxed4(su + 4 * idx[j]);
#pragma unroll
    for (int j = 0; j < kN; ++j)
      if (((want >> j) & 1u) && v[j].x != kScoreEmpty && v[j].y != kScoreEmpty &&
          v[j].z != kScoreEmpty && v[j].w != kScoreEmpty)
        want &= ~(1u << j);
    if (!want) break;
    if (*abort) return false;
    if (global_timer_ns() - t0 > 2000000000ull) { *abort = 1; return false; }
    __nanosleep(200);
  }
  return true;
}

// This lane's slice of the group's queries: qr[g][e] = q[g][lane * D/32 + e].
template <typename T, int D, int G>
__device__ __forceinline__ void load_q_slice(const T* qb, int lane, float (&qr)[G][D / 32]) {
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < D / 32; ++e) qr[g][e] = ldf(qb, g * D + lane * (D / 32) + e);
}

// max_g |q_g|_2 from every lane's slice (fp64 sums, a butterfly; the same in every lane).
template <int D, int G>
__device__ __forceinline__ double q_norm_max(const float (&qr)[G][D / 32]) {
  double best = 0.0;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) ss = fma((double)qr[g][e], (double)qr[g][e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    best = fmax(best, sqrt(ss));
  }
  return best;
}

// Twice a bound on |fl32(q . L) - q . L| for every row with |L|_2 <= lmax: gamma_D *
// sum|q_i L_i| <= gamma_D |q|_2 |L|_2 (FMA accumulation of D exact-input products), with
// margins for the fp32 norm itself and for the fp64 re-score.
template <int D>
__device__ __forceinline__ double score_error_window(double qmax, double lmax) {
  const double u = 5.9604644775390625e-8;   // 2^-24
  const double gam = D * u / (1.0 - D * u);
  const double w = 2.0 * (gam * 1.001 + 1e-12) * qmax * lmax + 1e-300;
  return w < INFINITY ? w : INFINITY;   // non-finite inputs: everything is in the window
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
  const int b = p / dm.H, h = p % dm.H;
  const T* qb = (const T*)a.q + ((size_t)b * dm.Hq + (size_t)h * G) * D;
  const T* L = (const T*)a.landmark + (size_t)p * Nc * D;

  const float lmax = __ldg(a.landmark_norm + p);
  float qr[G][D / 32];
  load_q_slice<T, D, G>(qb, g.tid & 31, qr);
  const uint32_t tk = group_kth_largest(
      g, Nc, k, [&](int i) { return f2key(__ldcg(s + i)); }, ms->hist, ms->bc);
  const double tau = (double)key2f(tk);
  const double delta = score_error_window<D>(q_norm_max<D, G>(qr), (double)lmax);
  const double hi = tau + delta, lo = tau - delta;
  if (g.tid == 0) ms->cnt = 0;
  g.sync();
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

// fp64 scores of window rows by one warp: lane l holds D/32 consecutive elements of
// each row and the same slice of each query head (qr); exact products, fp64 sums
// (lane-serial, then a butterfly); lane 0's value is stored. The loads of up to 8 rows
// are issued together.
template <typename T, int D, int G>
__device__ void score64_rows_warp(const T* Lp, const float (&qr)[G][D / 32], const int* wl,
                                  int w, int first, int stride, double* s64, int lane) {
  constexpr int E = D / 32;
  constexpr int kBatch = 8;
  for (int r0 = first; r0 < w; r0 += stride * kBatch) {
    float lv[kBatch][E];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = r0 + j * stride;
      if (i < w) {
        const T* row = Lp + (size_t)wl[i] * D;
#pragma unroll
        for (int e = 0; e < E; ++e) lv[j][e] = ldf(row, lane * E + e);
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = r0 + j * stride;
      if (i >= w) break;
      double best = -INFINITY;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        double acc = 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e) acc = fma((double)qr[g][e], (double)lv[j][e], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        best = fmax(best, acc);
      }
      if (lane == 0) s64[i] = best;
    }
  }
}

// A prefix of the k-th largest (1 <= k <= n) of n uint32 keys, exact in (at least) its
// top 8 * kPasses bits, the bits below the last resolved digit returned as zero. The bits
// that all n keys share (above the highest bit where the smallest and the largest key
// differ) are taken at once; 8-bit radix passes (most significant digit first) resolve
// the rest, so at most kPasses passes run and usually one fewer. Two histograms
// alternate: the one for pass p + 1 is cleared during pass p.
template <int kPasses, typename KeyFn>
__device__ uint32_t kth_largest_prefix(const Grp& g, int n, int k, KeyFn key_of, Misc* ms) {
  const int lane = g.tid & 31;
  for (int i = g.tid; i < 512; i += g.nt) ms->hist[i] = 0u;
  if (g.tid == 0) {
    ms->kr[0] = 0xFFFFFFFFu;
    ms->kr[1] = 0u;
  }
  g.sync();
  {
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i = g.tid; i < n; i += g.nt) {
      const uint32_t key = key_of(i);
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      atomicMin(&ms->kr[0], kmin);
      atomicMax(&ms->kr[1], kmax);
    }
  }
  g.sync();
  const uint32_t kmin = ms->kr[0], diff = kmin ^ ms->kr[1];
  const int lb = 32 - 8 * kPasses;                  // lowest bit that must be resolved
  int hi = diff ? 31 - __clz(diff) : -1;             // highest bit not shared by all keys
  const uint32_t common = hi < 0 ? 0xFFFFFFFFu : (hi >= 31 ? 0u : ~((2u << hi) - 1u));
  uint32_t prefix = kmin & common, mask = common;
  unsigned remaining = (unsigned)k;
  for (int pass = 0; hi >= lb; ++pass) {
    const int shift = hi - 7;                        // >= 0: hi >= lb >= 8
    unsigned* hist = ms->hist + 256 * (pass & 1);
    if (pass >= 1)
      for (int i = g.tid; i < 256; i += g.nt) ms->hist[256 * ((pass + 1) & 1) + i] = 0u;
    for (int i = g.tid; i < n; i += g.nt) {
      const uint32_t key = key_of(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    g.sync();
    if (g.tid < 32) {
      unsigned own = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) own += hist[255 - 8 * lane - j];
      unsigned incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const unsigned before = incl - own;
      if (before < remaining && incl >= remaining) {
        unsigned acc = before;
        for (int j = 0; j < 8; ++j) {
          const int dg = 255 - 8 * lane - j;
          const unsigned c = hist[dg];
          if (acc + c >= remaining) { ms->bc[2 * (pass & 1)] = (unsigned)dg; ms->bc[2 * (pass & 1) + 1] = remaining - acc; break; }
          acc += c;
        }
      }
    }
    g.sync();
    prefix |= ms->bc[2 * (pass & 1)] << shift;
    mask |= 255u << shift;
    remaining = ms->bc[2 * (pass & 1) + 1];
    hi = shift - 1;
  }
  return prefix;
}

// Fast path (see the file comment); needs k <= cap/2 and N_c <= kBitmapChunks. Reads each
// entry through a poll that waits out the sentinel, so it needs no separate wait for the
// pair. Expects ms->cnt, n_in, nwin and fmax at zero. Returns 1 when done; 0, having
// written no output, when the candidate set cannot be proven to hold the answer (every
// entry has been seen by then); -1 when a wait gave up.
template <typename T, int D, int G>
__device__ int select_pair_fast(const Grp& g, const SelectArgs& a, int p, float* ckey,
                                int* cid, uint32_t* bits, Misc* ms, volatile int* abort) {
  constexpr int kCap = cand_cap(G, D);
  constexpr int kB = 8;   // independent loads in flight per thread
  const Dims& dm = a.dm;
  const int Nc = dm.Nc, k = dm.k;
  const int lane = g.tid & 31;
  const uint32_t* su = reinterpret_cast<const uint32_t*>(a.scores + (size_t)p * Nc);
  const T* qb = (const T*)a.q + ((size_t)(p / dm.H) * dm.Hq + (size_t)(p % dm.H) * G) * D;
  const uint64_t t_start = global_timer_ns();
  double qmax;   // max_g |q_g|_2, for the error window
  {
    float qr[G][D / 32];
    load_q_slice<T, D, G>(qb, lane, qr);
    qmax = q_norm_max<D, G>(qr);
  }
  const int nw = (Nc + 31) >> 5;
  for (int i = g.tid; i < nw; i += g.nt) bits[i] = 0u;
  bool good = true;
  int m;
  float t0 = -INFINITY;
  const bool sampled = Nc > kCap;
  if (!sampled) {
    for (int base = 0; base < Nc; base += kB * g.nt) {
      int idx[kB];
      uint32_t want = 0, v[kB];
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        idx[j] = base + j * g.nt + g.tid;
        if (idx[j] < Nc) want |= 1u << j;
      }
      good = good && poll_words<kB>(su, idx, want, v, abort, t_start);
#pragma unroll
      for (int j = 0; j < kB; ++j)
        if ((want >> j) & 1u) {
          ckey[idx[j]] = __uint_as_float(v[j]);
          cid[idx[j]] = idx[j];
        }
    }
    if (!good) ms->cnt = -1;
    g.sync();
    if (ms->cnt < 0) return -1;
    m = Nc;
  } else {
    uint32_t* skey = reinterpret_cast<uint32_t*>(cid);
    for (int base = 0; base < kSample; base += kB * g.nt) {
      int idx[kB];
      uint32_t want = 0, v[kB];
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        const int i = base + j * g.nt + g.tid;
        idx[j] = (int)(((long long)i * Nc) / kSample);
        if (i < kSample) want |= 1u << j;
      }
      good = good && poll_words<kB>(su, idx, want, v, abort, t_start);
#pragma unroll
      for (int j = 0; j < kB; ++j)
        if ((want >> j) & 1u) skey[base + j * g.nt + g.tid] = f2key(__uint_as_float(v[j]));
    }
    if (!good) ms->cnt = -1;
    g.sync();
    if (ms->cnt < 0) return -1;
    int j = (int)((3LL * k * kSample) / (2LL * Nc)) + 16;
    if (j > kSample) j = kSample;
    t0 = key2f(kth_largest_prefix<2>(g, kSample, j, [&](int i) { return skey[i]; }, ms));
    // every score >= t0 becomes a candidate. Each thread polls 8 independent 16-byte
    // groups (4 scores; single scores when 4 does not divide N_c), keeps a mask of its
    // candidates, and one warp scan and one shared atomic per warp place them.
    const bool vec = (Nc & 3) == 0 && (reinterpret_cast<uintptr_t>(su) & 15) == 0;
    const int per = vec ? 4 : 1;   // scores per polled group
    const int n_groups = Nc / per;
    for (int base = 0; base < n_groups; base += kB * g.nt) {
      int idx[kB];
      uint32_t want = 0;
      uint4 v[kB];
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        idx[j] = base + j * g.nt + g.tid;
        if (idx[j] < n_groups) want |= 1u << j;
      }
      if (vec) {
        good = good && poll_vec4<kB>(su, idx, want, v, abort, t_start);
      } else {
        uint32_t v1[kB];
        good = good && poll_words<kB>(su, idx, want, v1, abort, t_start);
        const uint32_t ninf = __float_as_uint(-INFINITY);
#pragma unroll
        for (int j = 0; j < kB; ++j) v[j] = make_uint4(v1[j], ninf, ninf, ninf);
      }
      uint32_t keep = 0;   // bit 4j + e: score per * idx[j] + e
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        if (!((want >> j) & 1u)) continue;
        keep |= (__uint_as_float(v[j].x) >= t0 ? 1u : 0u) << (4 * j);
        keep |= (__uint_as_float(v[j].y) >= t0 ? 1u : 0u) << (4 * j + 1);
        keep |= (__uint_as_float(v[j].z) >= t0 ? 1u : 0u) << (4 * j + 2);
        keep |= (__uint_as_float(v[j].w) >= t0 ? 1u : 0u) << (4 * j + 3);
      }
      const int c = __popc(keep);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int wb = 0;
      if (lane == 31 && incl > 0) wb = atomicAdd(&ms->cnt, incl);
      wb = __shfl_sync(0xffffffffu, wb, 31);
      if (keep == 0) continue;
      int pos = wb + incl - c;
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        const uint32_t xs[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((keep >> (4 * j + e)) & 1u) {
            if (pos < kCap) { ckey[pos] = __uint_as_float(xs[e]); cid[pos] = per * idx[j] + e; }
            ++pos;
          }
        }
      }
    }
    if (!good) ms->n_in = -1;
  }
  g.sync();
  if (ms->n_in < 0) return -1;
  if (sampled) {
    m = ms->cnt;
    if (m > kCap || m < k) return 0;
  }
  const uint32_t tp = kth_largest_prefix<3>(g, m, k, [&](int i) { return f2key(ckey[i]); }, ms);
  const double tau_lo = (double)key2f(tp), tau_hi = (double)key2f(tp | 0xFFu);
  if (!(tau_lo <= tau_hi)) return 0;   // a non-finite bucket
  const double delta = score_error_window<D>(qmax, (double)__ldg(a.landmark_norm + p));
  const double hi = tau_hi + delta, lo = tau_lo - delta;
  if (sampled && (double)t0 > lo) return 0;   // the window may reach below the filter
  // classify: clearly in -> bitmap; window -> list (warp-aggregated counts)
  int* wl = ms->wl;
  for (int base = 0; base < m; base += g.nt) {
    const int i = base + g.tid;
    const double x = i < m ? (double)ckey[i] : -INFINITY;
    const bool in = i < m && x > hi;
    const bool win = i < m && !in && x >= lo;
    const unsigned bin = __ballot_sync(0xffffffffu, in), bwin = __ballot_sync(0xffffffffu, win);
    if (in) atomicOr(&bits[cid[i] >> 5], 1u << (cid[i] & 31));
    if (lane == 0 && bin) atomicAdd(&ms->n_in, __popc(bin));
    if (bwin) {
      int wb = 0;
      if (lane == 0) wb = atomicAdd(&ms->nwin, __popc(bwin));
      wb = __shfl_sync(0xffffffffu, wb, 0);
      const int pos = wb + __popc(bwin & ((1u << lane) - 1u));
      if (win && pos < kWindowCap) wl[pos] = cid[i];
    }
  }
  g.sync();
  const int n_in = ms->n_in, w = ms->nwin, need = k - n_in;
  if (w > kWindowCap) return 0;
  // window: when it holds exactly the rows still needed (the usual case: the k-th row
  // alone) all are in. Otherwise one warp per row re-scores in fp64 (queries as stored)
  // and the rows are ranked by (score desc, index asc).
  if (w == need) {
    for (int i = g.tid; i < w; i += g.nt) atomicOr(&bits[wl[i] >> 5], 1u << (wl[i] & 31));
    g.sync();
  } else if (w > 0) {
    const T* Lp = (const T*)a.landmark + (size_t)p * Nc * D;
    double* s64 = reinterpret_cast<double*>(ckey);   // candidates are no longer needed
    float qr[G][D / 32];
    load_q_slice<T, D, G>(qb, lane, qr);
    score64_rows_warp<T, D, G>(Lp, qr, wl, w, g.tid >> 5, g.nt >> 5, s64, lane);
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
  }
  // ascending output: each thread owns a run of bitmap words; one scan of their counts
  int32_t* sel = a.sel + (size_t)p * k;
  const int wpt = (nw + g.nt - 1) / g.nt;
  int cnt = 0;
  for (int j = 0; j < wpt; ++j) {
    const int wi = g.tid * wpt + j;
    if (wi < nw) cnt += __popc(bits[wi]);
  }
  int total;
  int pos = group_exclusive_scan(g, cnt, ms->iscr, &total);
  for (int j = 0; j < wpt; ++j) {
    const int wi = g.tid * wpt + j;
    uint32_t rem = wi < nw ? bits[wi] : 0u;
    while (rem) {
      const int bit = __ffs(rem) - 1;
      rem &= rem - 1;
      if (pos < k) sel[pos] = wi * 32 + bit;
      ++pos;
    }
  }
  return 1;
}

// Selects (b, h) pair p from its scores, waiting for them as it reads; leaves the scratch
// counters at zero. Returns false if a wait gave up.
template <typename T, int D, int G>
__device__ bool select_pair(const Grp& g, const SelectArgs& a, int p, float* ckey, int* cid,
                            uint32_t* bits, Misc* ms, volatile int* abort) {
  constexpr int kCap = cand_cap(G, D);
  const int Nc = a.dm.Nc, k = a.dm.k;
  const uint32_t* su = reinterpret_cast<const uint32_t*>(a.scores + (size_t)p * Nc);
  int r = 0;   // 1 done, 0 radix path, -1 gave up
  if (k < Nc && k <= kCap / 2 && Nc <= kBitmapChunks) {
    r = select_pair_fast<T, D, G>(g, a, p, ckey, cid, bits, ms, abort);
  } else {
    if (!wait_scores(g, su, Nc, abort)) ms->n_in = -1;   // every score, before any is used
    g.sync();
    r = ms->n_in < 0 ? -1 : 0;
    if (r == 0 && k >= Nc) {
      int32_t* sel = a.sel + (size_t)p * k;
      for (int i = g.tid; i < Nc; i += g.nt) sel[i] = i;
      r = 1;
    }
  }
  g.sync();
  if (r == 0) select_pair_radix<T, D, G>(g, a, p, ms);
  g.sync();
  if (g.tid == 0) { ms->cnt = 0; ms->n_in = 0; ms->nwin = 0; ms->fmax = 0.f; }
  g.sync();
  return r >= 0;
}

// ---------------------------------------------------------------- scoring
// Score of landmark row r of a swizzled fp32 stage (one row per lane).
template <int D, int G>
__device__ __forceinline__ float score_row_f32(const uint8_t* stage, int r, const float* sQ) {
  using Gm = Geom<float, D>;
  float2 acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < Gm::kChunks; ++c) {
    const int box = c >> 3, cc = c & 7;
    const uint4 w = *reinterpret_cast<const uint4*>(
        stage + box * Gm::kLps * 128 + r * 128 + ((cc ^ (r & 7)) << 4));
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
  float best = acc[0].x + acc[0].y;
#pragma unroll
  for (int g = 1; g < G; ++g) best = fmaxf(best, acc[g].x + acc[g].y);
  return best;
}

// Position in a stage's query block of dim d of a head (bf16 landmarks): the upper half
// of the dims has its 16-byte units XOR 4, so the two lanes of a pair in score_rows_pair,
// which read the lower and the upper half at the same step, hit different banks.
template <int D>
__device__ __forceinline__ int q_pos(int d) {
  return d < D / 2 ? d : ((((d >> 2) ^ 4) << 2) | (d & 3));
}

// Scores of rows r0 and r1 of a bf16 stage by a pair of lanes (lane half hh = lane & 1):
// each lane sums its half of the dims for both rows, so every query load feeds two rows
// (half the query traffic of one row per lane), and one shuffle per head and row adds the
// partner's half. The upper half walks its 16-byte chunks in XOR-4 order so the pair's
// landmark loads fall in different banks as well. Returns (score r0, score r1), the same
// in both lanes (fp32 addition commutes).
template <int D, int G>
__device__ __forceinline__ float2 score_rows_pair(const uint8_t* stage, int r0, int r1, int hh,
                                                  const float* sQ) {
  using Gm = Geom<__nv_bfloat16, D>;
  constexpr int H = Gm::kChunks / 2;   // 16-byte chunks per half row: 8 (D 128), 4 (D 64)
  float2 a0[G], a1[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    a0[g] = make_float2(0.f, 0.f);
    a1[g] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int st = 0; st < H; ++st) {
    const int c = hh * H + ((H == 8 && hh) ? (st ^ 4) : st);   // chunk: dims 8c .. 8c + 7
    const int box = c >> 3, cc = c & 7;
    const uint8_t* bp = stage + box * Gm::kLps * 128;
    const uint4 w0 = *reinterpret_cast<const uint4*>(bp + r0 * 128 + ((cc ^ (r0 & 7)) << 4));
    const uint4 w1 = *reinterpret_cast<const uint4*>(bp + r1 * 128 + ((cc ^ (r1 & 7)) << 4));
    const float2 v0 = bf2_to_f2(w0.x), v1 = bf2_to_f2(w0.y), v2 = bf2_to_f2(w0.z), v3 = bf2_to_f2(w0.w);
    const float2 u0 = bf2_to_f2(w1.x), u1 = bf2_to_f2(w1.y), u2 = bf2_to_f2(w1.z), u3 = bf2_to_f2(w1.w);
    const int qa = q_pos<D>(8 * c), qb = q_pos<D>(8 * c + 4);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 q0 = *reinterpret_cast<const float4*>(sQ + g * D + qa);
      const float4 q1 = *reinterpret_cast<const float4*>(sQ + g * D + qb);
      a0[g] = __ffma2_rn(make_float2(q0.x, q0.y), v0, a0[g]);
      a1[g] = __ffma2_rn(make_float2(q0.x, q0.y), u0, a1[g]);
      a0[g] = __ffma2_rn(make_float2(q0.z, q0.w), v1, a0[g]);
      a1[g] = __ffma2_rn(make_float2(q0.z, q0.w), u1, a1[g]);
      a0[g] = __ffma2_rn(make_float2(q1.x, q1.y), v2, a0[g]);
      a1[g] = __ffma2_rn(make_float2(q1.x, q1.y), u2, a1[g]);
      a0[g] = __ffma2_rn(make_float2(q1.z, q1.w), v3, a0[g]);
      a1[g] = __ffma2_rn(make_float2(q1.z, q1.w), u3, a1[g]);
    }
  }
  float best0 = -INFINITY, best1 = -INFINITY;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float z0 = a0[g].x + a0[g].y, z1 = a1[g].x + a1[g].y;
    z0 += __shfl_xor_sync(0xffffffffu, z0, 1);
    z1 += __shfl_xor_sync(0xffffffffu, z1, 1);
    best0 = fmaxf(best0, z0);
    best1 = fmaxf(best1, z1);
  }
  return make_float2(best0, best1);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kSelThreads, 1)
score_select_kernel(const SelectArgs a, const __grid_constant__ CUtensorMap lmap) {
  using Gm = Geom<T, D>;
  constexpr int kQ = G * D;        // query values per (b, h); a multiple of 32
  constexpr int kQL = kQ / 32;     // per producer lane
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
  int* stage_unit = reinterpret_cast<int*>(gbase + L.hdr);   // [kStages]; -2: no more
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L.bar + 8 * 2 * kStages);
  auto full = [&](int s) { return base + L.bar + 8u * (uint32_t)s; };
  auto empty = [&](int s) { return base + L.bar + 8u * (uint32_t)(kStages + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Nc = dm.Nc, P = dm.B * dm.H;
  const int upp = select_stages_per_pair(dm);   // stages of Gm::kLps rows per (b, h)
  const int U = P * upp;
  int* grab = a.counters;        // next stage to hand out
  int* exits = a.counters + 1;   // CTAs finished
  int* q_head = a.counters + 2;  // next (b, h) to select

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 32);                 // the producer warp's lanes
      mbar_init(empty(s), kConsumers / 32);   // one arrival per consumer warp
    }
    fence_mbar_init();
    ms->cnt = 0;
    ms->n_in = 0;
    ms->nwin = 0;
    ms->fmax = 0.f;
    ms->carry = -1;
  }
  __syncthreads();
  // a programmatic dependent (the reconstruct-and-attend kernel) may start as SMs free
  // up; it reads a pair's selection only after that pair's ready flag is set
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer warp
    // Lane 0 takes stages two fills ahead and issues their loads; every lane loads the
    // queries of the next fill's (b, h) one fill ahead and stages them.
    int last_i[kStages];
    for (int s = 0; s < kStages; ++s) last_i[s] = -1;
    bool ok = true;
    auto load_q = [&](int unit, float* qv) {
      const int pair = unit / upp;
      const T* qb = (const T*)a.q + ((size_t)(pair / dm.H) * dm.Hq + (size_t)(pair % dm.H) * G) * D;
#pragma unroll
      for (int j = 0; j < kQL; ++j) qv[j] = ldf(qb, lane + 32 * j);
    };
    // u: this fill's stage, un: the next one; lane 0's grab_pend is the take for the fill
    // after that, issued one fill earlier and read one fill later.
    int u = U, un = U, grab_pend = U;
    if (lane == 0) {
      u = atomicAdd(grab, 1);
      if (u < U) un = atomicAdd(grab, 1);
      if (un < U) grab_pend = atomicAdd(grab, 1);
    }
    u = __shfl_sync(0xffffffffu, u, 0);
    un = __shfl_sync(0xffffffffu, un, 0);
    float qa[kQL], qb[kQL];
    if (u < U) load_q(u, qa);
    int i = 0;
    // One fill; qc holds this fill's queries, qn receives the next fill's. Returns 0 to go
    // on, 1 when no stages are left (fill i's slot is free), 2 on a failed wait.
    auto step = [&](float (&qc)[kQL], float (&qn)[kQL]) -> int {
      const int s = i % kStages;
      int okw = 1;
      if (lane == 0) okw = mbar_wait_bounded(empty(s), ((i / kStages) & 1) ^ 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, okw, 0)) return 2;
      if (u >= U) return 1;   // slot s is free for the closing fill
      float* q_s = sQ + s * kQ;
#pragma unroll
      for (int j = 0; j < kQL; ++j) {
        const int f = lane + 32 * j;   // head f / D, dim f % D
        if constexpr (sizeof(T) == 2)
          q_s[(f / D) * D + q_pos<D>(f % D)] = qc[j];
        else
          q_s[f] = qc[j];
      }
      if (lane == 0) {
        stage_unit[s] = u;
        const int pair = u / upp, st = u % upp;
        const int row = pair * Nc + st * Gm::kLps;
        mbar_arrive_expect_tx(full(s), (uint32_t)(Gm::kBoxes * Gm::kLps * 128));
        for (int bx = 0; bx < Gm::kBoxes; ++bx)
          tma_load_2d(base + L.stages + s * kStageBytes + bx * Gm::kLps * 128, &lmap,
                      bx * Gm::kBoxCols, row, full(s));
        last_i[s] = i;
      } else {
        mbar_arrive(full(s));
      }
      // the next fill's queries and the take after the next
      if (un < U) load_q(un, qn);
      int unn = U;
      if (lane == 0 && un < U) {
        unn = grab_pend;
        grab_pend = unn < U ? atomicAdd(grab, 1) : U;
      }
      u = un;
      un = __shfl_sync(0xffffffffu, unn, 0);
      ++i;
      return 0;
    };
    for (;;) {
      int r = step(qa, qb);
      if (r == 0) r = step(qb, qa);
      if (r == 0) continue;
      ok = r == 1;
      break;
    }
    if (ok) {   // closing fill: no stages left
      const int s = i % kStages;
      if (lane == 0) stage_unit[s] = -2;
      mbar_arrive(full(s));
    }
    if (lane == 0 && *abort_flag) {   // loads may still be in flight: let them land
      for (int s = 0; s < kStages; ++s) {
        if (last_i[s] < 0) continue;
        int dummy = 0;
        mbar_wait_bounded(full(s), (last_i[s] / kStages) & 1, (volatile int*)&dummy);
      }
    }
  } else if (warp < kConsumers / 32) {
    // ------------------------------------------------------------ consumers
    const int tid = threadIdx.x;
    for (int i = 0;; ++i) {
      const int s = i % kStages;
      const bool okw = mbar_wait_bounded(full(s), (i / kStages) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, okw)) break;
      const int u = stage_unit[s];
      if (u < 0) break;
      const int pair = u / upp, st = u % upp;
      if constexpr (sizeof(T) == 2) {
        // lanes 2i, 2i + 1 score rows i and i + kLps/2 of the stage (kLps == 256 threads)
        static_assert(Gm::kLps == kConsumers, "one lane pair per two rows");
        const int hh = tid & 1, r0 = tid >> 1, r1 = r0 + Gm::kLps / 2;
        const float2 sc = score_rows_pair<D, G>(gbase + L.stages + s * kStageBytes, r0, r1, hh,
                                                sQ + s * kQ);
        const int c = st * Gm::kLps + (hh ? r1 : r0);
        if (c < Nc) a.scores[(size_t)pair * Nc + c] = hh ? sc.y : sc.x;
      } else {
        const int c = st * Gm::kLps + tid;
        if (tid < Gm::kLps && c < Nc)
          a.scores[(size_t)pair * Nc + c] =
              score_row_f32<D, G>(gbase + L.stages + s * kStageBytes, tid, sQ + s * kQ);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
    }
  }
  if (warp != kConsumers / 32) {
    // ------------------------------------------------------------ selection
    // The selection warps take the next (b, h), wait until all of its stages are handed
    // out and all of its scores have landed, select, and restore the sentinel; one
    // verdict per step for the whole group keeps its barrier sequence uniform. A pair
    // whose scoring ends in the last wave of stages (about the last `waves` stages of
    // every CTA) is not selected by these three warps: it is handed over, claimed, to the
    // consumers and the selection warps together (all but the producer), who meet once
    // the consumers have no stages left and select it several times faster right when
    // its last scores land, then any pairs still in the queue. The selection warps also
    // hand over (with no pair) when the queue is empty, so the meeting always happens.
    const bool sel_warp = warp > kConsumers / 32;
    const int waves = Nc > kLongPair ? kLateWavesLong : kLateWaves;
    const long long late_from = (long long)U - (long long)waves * gridDim.x;
    bool joined = !sel_warp;
    if (!sel_warp) named_bar_sync(kJoinBar, kConsumers + kSelectors);
    for (;;) {
      const Grp g = joined ? Grp{(int)threadIdx.x < kConsumers ? (int)threadIdx.x
                                                               : (int)threadIdx.x - 32,
                                 kConsumers + kSelectors, kJoinBar}
                           : Grp{(int)threadIdx.x - (kConsumers + 32), kSelectors, 2};
      if (g.tid == 0) {
        int pair = -1;
        if (joined && ms->carry >= 0) {
          pair = ms->carry;
          ms->carry = -1;
        } else if (!joined || !*abort_flag) {
          const int at = atomicAdd(q_head, 1);
          if (at < P && wait_counter_ge(grab, (at + 1) * upp, abort_flag)) pair = at;
        }
        ms->req = pair;
      }
      g.sync();
      const int pair = ms->req;
      g.sync();
      if (!joined && (pair < 0 || (long long)(pair + 1) * upp > late_from)) {
        if (g.tid == 0) ms->carry = pair;
        named_bar_sync(kJoinBar, kConsumers + kSelectors);
        joined = true;
        continue;
      }
      if (pair < 0) break;
      // a failed wait has raised the abort flag: the next step ends the loop
      if (!select_pair<T, D, G>(g, a, pair, ckey, cidv, bits, ms, abort_flag)) continue;
      if (a.ready && g.tid == 0) {   // select_pair ended on a group barrier
        __threadfence();
        const int b = pair / dm.H, hh = pair % dm.H;
        or_release(a.ready + ready_word(dm, b, hh), 1u << (b & 31));
      }
      // the sentinel goes back after the flag: only the next launch reads these scores
      clear_scores(g, reinterpret_cast<uint32_t*>(a.scores + (size_t)pair * Nc), Nc);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*abort_flag) raise_status(a.status, kStatusTimeout);
    // the last CTA out resets the counters and, after a failure, every score
    __threadfence();
    const bool last = atomicAdd(exits, 1) == (int)gridDim.x - 1;
    bool failed = false;
    if (last) {
      __threadfence();
      failed = *(volatile int*)a.status != 0;
      atomicExch(grab, 0);
      atomicExch(q_head, 0);
      atomicExch(exits, 0);
    }
    ms->req = failed ? 1 : 0;
  }
  __syncthreads();
  if (ms->req) {
    const Grp all{(int)threadIdx.x, (int)blockDim.x, 0};
    clear_scores(all, reinterpret_cast<uint32_t*>(a.scores), P * Nc);
  }
}

template <typename T, int D, int G>
cudaError_t launch_typed(const SelectArgs& a, int num_sms, cudaStream_t s) {
  using Gm = Geom<T, D>;
  CUtensorMap map;
  if (!make_tensor_map_2d(&map, a.landmark, a.dm.dtype, (uint64_t)D,
                          (uint64_t)a.dm.B * a.dm.H * a.dm.Nc, Gm::kBoxCols, Gm::kLps, 128,
                          256))
    return cudaErrorInvalidValue;
  const SelSmem L = sel_smem(G, D);
  if (L.total > (uint32_t)kSmemLimit) return cudaErrorInvalidValue;
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
