// ssa_fwd.cu -- skip-softmax / N:M sparse flash-attention forward for B200
// (sm_100a), and the C ABI declared in include/ssa.h.
//
// Method (cited by page title and section):
//   "Skip-Softmax Sparse Attention for Diffusion Models" (intro, "Threshold
//   Modes"): a KV tile whose scores are negligible is skipped; the kernel
//   compares against log2(lambda).  Rule: skip a (Br x Bc) tile when every
//   row has exp(tile_row_max - running_max) < lambda.
//   "Attention Sparsity for HuggingFace Models" ("N:M Sparse Softmax",
//   custom N:M configuration): per M consecutive keys keep the top-N scores,
//   the rest become -inf; sink and recent-window keys stay dense.
//
// One CTA owns two 128-row query tiles (A and B, adjacent in the sequence) of
// one (batch, query head) and walks the key tiles they can see; K and V tiles
// are loaded once for both.  Warp roles (384 threads):
//   warp 0      Q and K producer: TMA into a K ring (2 deep with 128 x 128
//               tiles of K and V; 4 deep where shared memory allows)
//   warp 1      TMEM owner and MMA issuer: S_t = Q_t K^T and O_t += P_t V on
//               tcgen05, ping-ponging between the two tiles so the tensor pipe
//               works on one tile while the other tile's softmax runs
//   warp 2      V producer: issues a V tile's TMA only once a tile has decided
//               to keep it, so a tile skipped by both never loads V
//   warps 4..7  softmax of tile A, warps 8..11 softmax of tile B: thread r
//               owns query row r (TMEM lane r): masks, N:M top-N in registers,
//               tile row max, skip vote, exp2, P -> TMEM, lazy O rescale,
//               epilogue
// TMEM (512 columns): tile t uses S/P at column 256 t and O at 256 t + 128.
// P (bf16, two per 32-bit column) overwrites the S columns it came from and
// is the A operand of the P.V MMA straight from TMEM.  Because S_t(j+1) is
// issued after O_t += P_t(j) V_j, the completion of S_t(j+1) also proves
// that every earlier P.V of tile t has finished, so the softmax may rescale
// O_t without another wait.
//
// When Br = 64 each 128-row tile carries two logical query tiles (rows 0-63
// and 64-127) that vote, count and keep state separately; P.V is issued when
// either keeps the key tile, with P = 0 for the half that skipped.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/ssa.h"
#include "internal.h"
#include "ptx.cuh"

namespace ssa {

constexpr int BM = 128;       // rows per query tile = tcgen05 M
constexpr int NQT = 2;        // query tiles per CTA
constexpr int RING_MAX = 4;   // deepest K and V rings (see Smem)
constexpr int NTHREADS = 384;
constexpr int TMEM_COLS = 512;
constexpr uint64_t WAIT_TIMEOUT_NS = 2000000000ull;  // default limit of a pipeline wait (2 s)
// Limit of the waits that make a failing CTA's own asynchronous work (TMA
// loads, MMAs) finish before it frees its memory; never shortened.
constexpr uint64_t DRAIN_TIMEOUT_NS = 2000000000ull;
constexpr float RESCALE_LOG2 = 8.0f;  // lazy O rescale once the max grew by 2^8
constexpr int VSLOTS = 4;             // vote slots per tile (see Bars::vote_bar)
// Key tiles a CTA can list when the caller selects key blocks by bitmap.
constexpr int MAX_LISTED_TILES = 2048;

struct Params {
  __nv_bfloat16* out;
  float* lse;
  int32_t* skip_count;
  uint32_t* skip_bits;  // optional
  uint32_t* keep_bits;  // optional
  int32_t* v_loads;     // optional [B, Hq, nPairs]: V tile loads each CTA issued
  int* status;
  int B, Hq, Hkv, Lq, Lk, causal, mode, n, m, sink, recent;
  int half;   // Br == 64
  int nQp;    // 128-row tiles per (b, hq)
  int nQ;     // logical query tiles per (b, hq)
  int nK;     // key tiles
  int nKw;    // words of skip bits per logical query tile
  int Lkw;    // words of keep bits per row
  float scale;
  float scale_log2;
  float log2_lambda;  // -inf for lambda == 0
  unsigned long long wait_ns;  // limit of each pipeline wait
  const uint32_t* block_mask;  // optional [B, Hkv, nQ, nKw]: key blocks each query block visits
  // proxy compensation of the omitted key blocks (bitmap variant only)
  int nP;       // proxy steps: summary rows of all nK blocks in chunks of Bc
  int n_last;   // keys in the final key block (its token mass)
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t k_full[RING_MAX], k_empty[RING_MAX];
  uint64_t v_full[RING_MAX], v_empty[RING_MAX];
  uint64_t s_full[NQT], p_half[NQT], p_ready[NQT], o_done[NQT];
  // A tile's votes of its i-th step (counting the steps it takes part in) sit
  // in slot i % VSLOTS (bytes and barrier phase i / VSLOTS).  A tile's softmax
  // runs at most two of its steps ahead of the V producer's read of its votes
  // (the V producer may still read tile B's byte of a step after its V load
  // released that step), so four slots never alias; two could.
  uint64_t vote_bar[NQT][VSLOTS];  // per tile and slot: one arrival per softmax warp
  uint64_t mma_done;
  uint32_t tmem_base;
  uint32_t vote[NQT][VSLOTS];      // byte w: softmax warp w of the tile keeps the key tile
  uint32_t abort_flag;
  int listed;                        // block-mask mode: key tiles in ktile[]
  int listed_t[NQT];                 // tile t takes part in no step from listed_t[t] on
  uint16_t ktile[MAX_LISTED_TILES];  // block-mask mode: the CTA's key tiles, ascending
  // block-mask mode: bit 2t + h of part[j] is set when logical query tile
  // (half) h of tile t selects and can see ktile[j]; tile t takes part in
  // step j when either of its bits is.  Each tile's barrier phases and vote
  // slots count only the steps it takes part in.
  uint8_t part[MAX_LISTED_TILES];
};

template <int D, int BC>
struct Smem {
  static constexpr uint32_t QT_BYTES = BM * D * 2;  // one query tile
  static constexpr uint32_t K_BYTES = BC * D * 2;
  static constexpr uint32_t V_BYTES = BC * D * 2;
  // K and V ring depths: four where both query tiles and four of each fit
  // (64-key tiles, or d = 64), else two.  A step of a 64-key tile is short, so
  // the loads need more steps of lead to hide their latency.
  static constexpr int KST = (NQT * QT_BYTES + RING_MAX * (K_BYTES + V_BYTES) + 16384 <= 227u * 1024u) ? RING_MAX : 2;
  static constexpr int VST = KST;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + NQT * QT_BYTES;
  static constexpr uint32_t V_OFF = K_OFF + KST * K_BYTES;
  static constexpr uint32_t BAR_OFF = V_OFF + VST * V_BYTES;
  static constexpr uint32_t TOTAL = BAR_OFF + ((sizeof(Bars) + 127) / 128) * 128;
  static constexpr uint32_t ALLOC = TOTAL + 1024;  // slack for 1024-byte alignment
  static_assert(ALLOC <= 227u * 1024u, "dynamic shared memory above the per-CTA limit");
};

// Key tiles visited by a logical query tile: all of them without a causal
// mask; otherwise up to the tile holding the key at the last row's position
// (bottom-right alignment), none when that position is negative.
__host__ __device__ inline int visited_key_tiles(int causal, int Lq, int Lk, int Br, int Bc, int qt) {
  const int nK = (Lk + Bc - 1) / Bc;
  if (!causal) return nK;
  long long last_row = (long long)qt * Br + Br - 1;
  if (last_row > Lq - 1) last_row = Lq - 1;
  const long long last_pos = last_row + (long long)Lk - Lq;
  if (last_pos < 0) return 0;
  const long long t = last_pos / Bc + 1;
  return t > nK ? nK : (int)t;
}

__device__ __forceinline__ float mufu_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void record_failure(const Params& p, Bars* bars) {
  *reinterpret_cast<volatile uint32_t*>(&bars->abort_flag) = 1u;
  atomicOr(p.status, 1);
}
__device__ __forceinline__ bool aborted(Bars* bars) {
  return *reinterpret_cast<volatile uint32_t*>(&bars->abort_flag) != 0u;
}

template <int N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Sorting networks (descending) used to find the N-th largest score of an
// N:M group: 5 comparators for 4 inputs, Batcher's odd-even merge sort (19
// comparators) for 8.
__device__ __forceinline__ void cmpx(float& hi, float& lo) {
  const float h = fmaxf(hi, lo), l = fminf(hi, lo);
  hi = h;
  lo = l;
}
template <int M>
__device__ __forceinline__ void sort_desc(float (&s)[M]) {
  if constexpr (M == 4) {
    cmpx(s[0], s[1]); cmpx(s[2], s[3]); cmpx(s[0], s[2]); cmpx(s[1], s[3]); cmpx(s[1], s[2]);
  } else {
    cmpx(s[0], s[1]); cmpx(s[2], s[3]); cmpx(s[4], s[5]); cmpx(s[6], s[7]);
    cmpx(s[0], s[2]); cmpx(s[1], s[3]); cmpx(s[1], s[2]);
    cmpx(s[4], s[6]); cmpx(s[5], s[7]); cmpx(s[5], s[6]);
    cmpx(s[0], s[4]); cmpx(s[1], s[5]); cmpx(s[2], s[6]); cmpx(s[3], s[7]);
    cmpx(s[2], s[4]); cmpx(s[3], s[5]);
    cmpx(s[1], s[2]); cmpx(s[3], s[4]); cmpx(s[5], s[6]);
  }
}

// N:M selection on one thread's row, 64 columns at a time: for each aligned
// group of M keys keep a key iff it is inside the sink / recent window or
// among the N largest scores of its group, equal scores ranked by lower
// index; dropped keys become -inf.  Masked keys are already -inf and stay
// -inf.  The fast form uses thr, the N-th largest score of a group, and nxt,
// the (N+1)-th: thr > nxt means the top N are exactly the keys >= thr
// (thr = -inf: every finite key).  It reports whether any group had an exact
// tie at the boundary (thr == nxt, finite); the caller then redoes the row
// from the original scores with explicit ranks.
// (bitwise, not short-circuit, logic throughout: the per-key decisions differ
// between lanes and must compile to predicated selects, not branches)
__device__ __forceinline__ bool in_window(int jj, int pos, int sink, int recent) {
  return (jj < sink) | ((unsigned)(pos - jj) < (unsigned)recent);
}

template <bool WIN>
__device__ __forceinline__ void nm_keep_group(float* v, int M, float thr, int col, int pos, int sink,
                                              int recent) {
#pragma unroll
  for (int a = 0; a < M; ++a) {
    bool keep = v[a] >= thr;
    if constexpr (WIN) keep |= in_window(col + a, pos, sink, recent);
    v[a] = keep ? v[a] : -INFINITY;
  }
}

// 4-wide groups, N fixed at compile time: order statistics from min/max.
// The tie test of the 2:4, 3:4 and 4:8 forms keeps the smallest gap t - nx
// over the groups: 0 exactly when some group has t == nx finite; a group with
// t = nx = -inf gives NaN, which fminf passes over.  (A spurious 0 could only
// send the warp to the exact rank-based redo, never to a wrong selection.)
// Measured: +3.4 % on 2:4, +4.5 % on skip + 2:4; the 1:4 and run-time-N
// 8-wide forms keep a predicate per group, which measured faster there.
template <int NN, bool WIN>
__device__ __forceinline__ bool nm4_fast(float (&x)[64], int col0, int pos, int sink, int recent) {
  float gap = INFINITY;
  bool tie = false;
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    float* v = &x[4 * g];
    const float hab = fmaxf(v[0], v[1]), lab = fminf(v[0], v[1]);
    const float hcd = fmaxf(v[2], v[3]), lcd = fminf(v[2], v[3]);
    const float mnh = fminf(hab, hcd), mxl = fmaxf(lab, lcd);
    float t;  // N-th largest, and its tie with the (N+1)-th
    if constexpr (NN == 1) {
      t = fmaxf(hab, hcd);
      const float nx = fmaxf(mnh, mxl);
      tie |= (t == nx) & (t != -INFINITY);
    } else if constexpr (NN == 2) {
      t = fmaxf(mnh, mxl);
      gap = fminf(gap, fabsf(mnh - mxl));
    } else {
      t = fminf(mnh, mxl);
      gap = fminf(gap, t - fminf(lab, lcd));
    }
    nm_keep_group<WIN>(v, 4, t, col0 + 4 * g, pos, sink, recent);
  }
  return NN == 1 ? tie : gap == 0.f;
}

// 8-wide groups: a sorting network per group.
template <bool WIN>
__device__ __forceinline__ bool nm8_fast(float (&x)[64], int N, int col0, int pos, int sink, int recent) {
  bool tie = false;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    float srt[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) srt[a] = x[8 * g + a];
    sort_desc<8>(srt);
    float t = srt[0], nx = srt[1];
#pragma unroll
    for (int r = 1; r < 8; ++r)
      if (N == r + 1) {  // uniform across the CTA
        t = srt[r];
        nx = r + 1 < 8 ? srt[r + 1] : -INFINITY;
      }
    tie |= (t == nx) & (t != -INFINITY);
    nm_keep_group<WIN>(&x[8 * g], 8, t, col0 + 8 * g, pos, sink, recent);
  }
  return tie;
}

// 8-wide groups with N = 4: the 4th and 5th largest of a group from its two
// sorted halves a, c (5 comparators each): the k-th largest of the union is
// the largest, over i + j = k, of min(i-th largest of a, j-th largest of c)
// (the 0-th being +inf).  32 min/max against 38 for a full sort plus the
// run-time choice of N.
template <bool WIN>
__device__ __forceinline__ bool nm8_n4(float (&x)[64], int col0, int pos, int sink, int recent) {
  float gap = INFINITY;  // see nm4_fast
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    float a[4], c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[i] = x[8 * g + i];
      c[i] = x[8 * g + 4 + i];
    }
    sort_desc<4>(a);
    sort_desc<4>(c);
    const float t = fmaxf(fmax3(c[3], fminf(a[0], c[2]), fminf(a[1], c[1])), fmaxf(fminf(a[2], c[0]), a[3]));
    const float nx = fmaxf(fmax3(fminf(a[0], c[3]), fminf(a[1], c[2]), fminf(a[2], c[1])), fminf(a[3], c[0]));
    gap = fminf(gap, t - nx);
    nm_keep_group<WIN>(&x[8 * g], 8, t, col0 + 8 * g, pos, sink, recent);
  }
  return gap == 0.f;
}

template <int M, bool WIN>
__device__ __forceinline__ bool nm_fast_w(float (&x)[64], int N, int col0, int pos, int sink, int recent) {
  if constexpr (M == 4) {
    switch (N) {  // uniform across the CTA
      case 1: return nm4_fast<1, WIN>(x, col0, pos, sink, recent);
      case 2: return nm4_fast<2, WIN>(x, col0, pos, sink, recent);
      case 3: return nm4_fast<3, WIN>(x, col0, pos, sink, recent);
      default: return false;  // N = 4 keeps every key
    }
  } else {
    return nm8_fast<WIN>(x, N, col0, pos, sink, recent);
  }
}

template <int M>
__device__ __forceinline__ bool nm_fast(float (&x)[64], int N, int col0, int pos, int sink, int recent,
                                        bool windows) {
  // windows is uniform across the CTA for a key tile
  return windows ? nm_fast_w<M, true>(x, N, col0, pos, sink, recent)
                 : nm_fast_w<M, false>(x, N, col0, pos, sink, recent);
}

// 4-wide groups with N fixed by the kernel instance: one copy of the
// selection instead of one per N (the softmax loop then fits the
// instruction cache; measured +4 % on 2:4 prefill, +7 % on 2:4 with skip).
template <int NN>
__device__ __forceinline__ bool nm4_fixed(float (&x)[64], int col0, int pos, int sink, int recent,
                                          bool windows) {
  return windows ? nm4_fast<NN, true>(x, col0, pos, sink, recent) : nm4_fast<NN, false>(x, col0, pos, sink, recent);
}

// Explicit ranks (the exact-tie path): rank = number of group keys that
// come first, a higher score or an equal score at a lower index.
template <int M>
__device__ __forceinline__ void nm_by_rank(float (&x)[64], int N, int col0, int pos, int sink,
                                           int recent, bool windows) {
#pragma unroll
  for (int g = 0; g < 64 / M; ++g) {
    int rank[M];
#pragma unroll
    for (int a = 0; a < M; ++a) rank[a] = 0;
#pragma unroll
    for (int a = 0; a < M; ++a)
#pragma unroll
      for (int c = a + 1; c < M; ++c) {
        if (x[g * M + c] > x[g * M + a]) ++rank[a];
        else ++rank[c];
      }
#pragma unroll
    for (int a = 0; a < M; ++a) {
      const bool keep = (rank[a] < N) | (windows & in_window(col0 + g * M + a, pos, sink, recent));
      x[g * M + a] = keep ? x[g * M + a] : -INFINITY;
    }
  }
}

// The exact-tie path of the N:M selection, out of line so that its registers
// do not burden the softmax loop: one row of S (columns [0, BC) at s_addr)
// from TMEM, the causal / length mask (columns past lim become -inf), the
// rank-based selection, and the selected scores written back over S, from
// where the caller reloads them.  Warp-collective (the caller's branch is
// warp-uniform).
template <int M, int BC>
__device__ __noinline__ void nm_redo_in_tmem(uint32_t s_addr, int N, int col0, int lim, int pos, int sink,
                                             int recent, bool windows) {
#pragma unroll 1
  for (int bb = 0; bb < BC / 64; ++bb) {
    float x[64];
    tmem_ld64f(s_addr + 64 * bb, x);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 64; ++i)
      if (64 * bb + i > lim) x[i] = -INFINITY;
    nm_by_rank<M>(x, N, col0 + 64 * bb, pos, sink, recent, windows);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t u[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(x[32 * h + i]);
      tmem_st32(s_addr + 64 * bb + 32 * h, u);
    }
  }
  tmem_wait_st();
}

struct Work {
  int b, hq, hkv;
  int pt[NQT];            // 128-row tile index of tile t
  int nvis_h[NQT][2];     // visited key tiles per logical half
  int nvis_t[NQT];        // per tile
  int nvis;               // per CTA
};

// NM_M: 0 no N:M; 8 eight-wide groups (N at run time); 84 eight-wide groups
// with N = 4; 41, 42, 43 four-wide groups with N = 1, 2, 3.
// VAR: 0 plain, 1 with debug outputs (skip / keep bits), 2 key blocks selected by
// bitmap, 3 key blocks selected by bitmap with proxy compensation of the others.
template <int D, int BC, int NM_M, int VAR>
__device__ __forceinline__ void softmax_tile(const Params& p, Bars* bars, int b, int hq, int hkv,
                                             int t, int pt, int nvis_h0, int nvis_h1, int nsteps,
                                             uint32_t tmem) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int row = tid - 128 - 128 * t;
  const int quarter = warp & 3;
  const int half = p.half ? (row >> 6) : 0;
  const int grow = pt * BM + row;
  const bool valid = grow < p.Lq;
  const int pos = grow + p.Lk - p.Lq;
  const int pos_first = pt * BM + p.Lk - p.Lq;
  const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
  const uint32_t s_col = 256 * t, o_col = 256 * t + 128;
  const bool skip_on = (p.mode & SSA_MODE_SKIP) != 0;
  constexpr bool nm_on = NM_M != 0;
  const bool leader = p.half ? ((row & 63) == 0) : (row == 0);
  const int my_nvis = half ? nvis_h1 : nvis_h0;
  constexpr bool DBG = VAR == 1, MASK = VAR >= 2, PROXY = VAR == 3;
  const int nvis = nsteps;  // = max(nvis_h0, nvis_h1) unless key blocks are selected by bitmap
  const int listed = MASK ? bars->listed : 0;  // exact steps, before the proxy steps
  const bool vote_on = skip_on || MASK;

  float m_true = -INFINITY;  // running max over kept tiles (raw q.k units)
  float m_ref = -INFINITY;   // reference the O accumulator and l are scaled to
  float l = 0.f;
  int n_pv = 0;
  int skipped = 0;
  uint32_t skip_word = 0;
  bool failed = false;

  int step = 0;  // steps this tile took part in: its barrier phases and vote slots
  for (int j = 0; j < nvis; ++j) {
    // key tile of this step, and whether each logical query tile (half) of
    // this tile visits it: visible, and selected when a bitmap is given.  A
    // proxy step g covers the summaries of key blocks [g Bc, g Bc + Bc).
    const bool is_proxy = PROXY && j >= listed;
    // with a bitmap, the tile takes part only in the listed steps it selects
    const uint32_t pbits = (MASK && !is_proxy) ? ((uint32_t)bars->part[j] >> (2 * t)) & 3u : 3u;
    if (pbits == 0u) continue;
    const int i_step = MASK ? step++ : j;
    bool ok = !failed && mbar_wait(smem_u32(&bars->s_full[t]), i_step & 1, p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    float m_tile = -INFINITY;
    const int kt = is_proxy ? j - listed : MASK ? (int)bars->ktile[j] : j;
    const int col0 = kt * BC;  // first key (exact step) or first key block (proxy step)
    auto visits = [&](int h) -> bool {
      const int nv = h ? nvis_h1 : nvis_h0;
      if constexpr (!MASK) {
        return j < nv;
      } else {
        if (is_proxy) return nv > 0;
        return (pbits >> (p.half ? h : 0)) & 1u;
      }
    };
    const bool vis0 = visits(0), vis1 = p.half ? visits(1) : vis0;
    const bool my_vis = half ? vis1 : vis0;
    // Pass 1: the whole row of S in registers -- masks, N:M, tile row max.
    // The scores stay in registers through the vote and become P in pass 2.
    const bool need_mask = (col0 + BC > p.Lk) || (p.causal && col0 + BC - 1 > pos_first);
    // does this key tile meet the sink or any row's recent window?
    const bool nm_windows = nm_on && ((col0 < p.sink) ||
                                      (col0 <= pos_first + BM - 1 && col0 + BC - 1 > pos_first - p.recent));
    float x[BC];
    // proxy step: the final key block's score (its token mass differs), -inf
    // when it is not in this chunk or is computed exactly
    float x_last = -INFINITY;
    // S from TMEM with the causal / length mask applied
    auto load_scores = [&]() {
#pragma unroll
      for (int c = 0; c < BC / 64; ++c) tmem_ld64f(lane_base + s_col + 64 * c, &x[64 * c]);
      const int c_last = p.nK - 1 - col0;
      if (is_proxy && c_last < BC) x_last = tmem_ld1f(lane_base + s_col + c_last);
      tmem_wait_ld();
      if (is_proxy) {
        // a block computed exactly by this query tile, or past the last
        // block, contributes no proxy
        const int qt = p.half ? 2 * pt + half : pt;
        const uint32_t* mw = p.block_mask + ((size_t)(b * p.Hkv + hkv) * p.nQ + (qt < p.nQ ? qt : 0)) * p.nKw;
#pragma unroll
        for (int w = 0; w < BC / 32; ++w) {
          const int wi = col0 / 32 + w;
          uint32_t drop = (qt < p.nQ && wi < p.nKw) ? mw[wi] : 0xffffffffu;
          const int left = p.nK - 32 * wi;  // blocks of this word that exist
          if (left < 32) drop |= left <= 0 ? 0xffffffffu : (0xffffffffu << left);
#pragma unroll
          for (int u = 0; u < 32; ++u)
            if ((drop >> u) & 1u) x[32 * w + u] = -INFINITY;
          if (c_last >= 32 * w && c_last < 32 * w + 32 && ((drop >> (c_last - 32 * w)) & 1u)) x_last = -INFINITY;
        }
        if (qt >= p.nQ) x_last = -INFINITY;
      } else if (need_mask) {
        // last visible column of this row, relative to the tile
        int lim = p.Lk - 1 - col0;
        if (p.causal && pos - col0 < lim) lim = pos - col0;
#pragma unroll
        for (int i = 0; i < BC; ++i)
          if (i > lim) x[i] = -INFINITY;
      }
    };
    if (ok) {
      tc_fence_after();
      load_scores();
      if constexpr (nm_on) {
        constexpr int MM = (NM_M == 8 || NM_M == 84) ? 8 : 4;  // group width
        bool tie = false;
#pragma unroll
        for (int bb = 0; bb < BC / 64; ++bb) {
          auto& xb = *reinterpret_cast<float(*)[64]>(&x[64 * bb]);
          if constexpr (NM_M == 84)
            tie |= nm_windows ? nm8_n4<true>(xb, col0 + 64 * bb, pos, p.sink, p.recent)
                              : nm8_n4<false>(xb, col0 + 64 * bb, pos, p.sink, p.recent);
          else if constexpr (NM_M >= 41 && NM_M <= 43)
            tie |= nm4_fixed<NM_M - 40>(xb, col0 + 64 * bb, pos, p.sink, p.recent, nm_windows);
          else
            tie |= nm_fast<MM>(xb, p.n, col0 + 64 * bb, pos, p.sink, p.recent, nm_windows);
        }
        if (__any_sync(0xffffffffu, tie)) {
          // an exact tie at a group boundary in some row of this warp: the
          // whole warp starts again from the scores (still in TMEM; the
          // tcgen05 accesses are warp-collective) and ranks explicitly.  With
          // 128-key tiles that runs out of line, leaving the selected scores
          // in place of S to be reloaded (inline, its registers made the
          // loop spill: measured +3 % on 2:4, +7 % on 4:8); 64-key tiles, and
          // the 1:4 instance (out of line it spills instead), redo it in
          // registers.
          if constexpr (BC == 128 && NM_M != 41) {
            int lim = BC - 1;
            if (need_mask) {
              lim = p.Lk - 1 - col0;
              if (p.causal && pos - col0 < lim) lim = pos - col0;
            }
            nm_redo_in_tmem<MM, BC>(lane_base + s_col, p.n, col0, lim, pos, p.sink, p.recent, nm_windows);
#pragma unroll
            for (int c = 0; c < BC / 64; ++c) tmem_ld64f(lane_base + s_col + 64 * c, &x[64 * c]);
            tmem_wait_ld();
          } else {
            load_scores();
#pragma unroll
            for (int bb = 0; bb < BC / 64; ++bb)
              nm_by_rank<MM>(*reinterpret_cast<float(*)[64]>(&x[64 * bb]), p.n, col0 + 64 * bb, pos,
                             p.sink, p.recent, nm_windows);
          }
        }
      }
      // four independent chains keep the dependent depth at BC / 8
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < BC; i += 8) {
        mx0 = fmax3(mx0, x[i], x[i + 1]);
        mx1 = fmax3(mx1, x[i + 2], x[i + 3]);
        mx2 = fmax3(mx2, x[i + 4], x[i + 5]);
        mx3 = fmax3(mx3, x[i + 6], x[i + 7]);
      }
      m_tile = fmaxf(fmax3(mx0, mx1, mx2), mx3);
      if (DBG && p.keep_bits != nullptr && valid && my_vis) {
        uint32_t* kb = p.keep_bits + ((size_t)(b * p.Hq + hq) * p.Lq + grow) * p.Lkw;
#pragma unroll
        for (int w = 0; w < BC / 32; ++w) {
          uint32_t word = 0;
#pragma unroll
          for (int u = 0; u < 32; ++u) word |= (x[32 * w + u] != -INFINITY ? 1u : 0u) << u;
          const int wi = col0 / 32 + w;
          if (wi < p.Lkw) kb[wi] = word;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < BC; ++i) x[i] = -INFINITY;
    }
    // A warp whose wait gave up keeps going with undefined data (so every
    // barrier and hand-off still pairs up) and keeps the tile; the failure
    // is already recorded.
    if (!ok && !failed && lane == 0) record_failure(p, bars);
    if (!ok) failed = true;
    const bool negligible =
        ok && (!valid || m_tile == -INFINITY ||
               (m_true != -INFINITY && (m_tile - m_true) * p.scale_log2 < p.log2_lambda));
    // The skip vote: each warp publishes one byte, "some row of mine keeps
    // the tile", and arrives on the tile's vote barrier for this step's
    // parity.  The MMA warp and the V producer read the same four bytes.
    const uint32_t vbar = smem_u32(&bars->vote_bar[t][i_step % VSLOTS]);
    bool wkeep = my_vis;
    if (vote_on) {
      wkeep = (skip_on ? !__all_sync(0xffffffffu, negligible) : true) && my_vis;
      if (lane == 0) {
        st_shared_u8(smem_u32(&bars->vote[t][i_step % VSLOTS]) + quarter, wkeep ? 1u : 0u);
        mbar_arrive(vbar);
      }
    }
    // keep_h[h]: logical query tile (half) h keeps this key tile
    bool keep_h[2] = {vis0, vis1};
    // (warp-uniform outcome: the tcgen05 accesses that follow are warp-collective)
    if (vote_on) {
      if (wkeep) {
        // A warp with a row that keeps the tile knows that its query tile
        // keeps it (the tile is skipped only if every row is negligible), so
        // it goes on at once; the other half's decision does not concern it.
        keep_h[0] = keep_h[1] = true;
      } else if (!__all_sync(0xffffffffu, mbar_wait(vbar, (i_step / VSLOTS) & 1, p.wait_ns))) {
        // only a warp whose rows are all negligible waits for the others' votes
        if (!failed && lane == 0) record_failure(p, bars);
        failed = true;  // and keeps the tile
      } else {
        const uint32_t w = ld_shared_u32(smem_u32(&bars->vote[t][i_step % VSLOTS]));
        keep_h[0] = p.half ? (w & 0xffffu) != 0u : w != 0u;
        keep_h[1] = p.half ? (w >> 16) != 0u : w != 0u;
      }
    }
    // "P of the first 64 keys is in TMEM" (one arrival per warp, every step)
    auto send_first_half = [&]() {
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_half[t]));
    };
    const bool mine = half ? keep_h[1] : keep_h[0];
    if (mine) {
      const float m_new = fmaxf(m_true, m_tile);
      bool resc = false;
      float m_ref_new = m_ref, alpha = 1.f;
      if (m_ref == -INFINITY) m_ref_new = m_new;  // first kept key: O and l are still zero
      else resc = (m_new - m_ref) * p.scale_log2 > RESCALE_LOG2;
      // O, when rescaled, is rescaled before this tile's P.V may start.
      const bool any_resc = __any_sync(0xffffffffu, resc);
      if (resc) {
        alpha = mufu_exp2((m_ref - m_new) * p.scale_log2);
        m_ref_new = m_new;
      }
      // Pass 2: P = exp2((s - m_ref) * scale * log2 e) from the registers
      // pass 1 left, 32 bf16 pairs per 64 columns
      const float c = p.scale_log2;
      const float mref_s = (m_ref_new == -INFINITY) ? 0.f : m_ref_new * c;
      const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-mref_s, -mref_s);
      uint64_t ls2 = f2_pack(0.f, 0.f);
      auto p_block = [&](int bb) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint64_t a2 = ffma2(f2_pack(x[64 * bb + 2 * i], x[64 * bb + 2 * i + 1]), c2, nm2);
          float a0, a1;
          f2_unpack(a2, a0, a1);
          const float p0 = mufu_exp2(a0), p1 = mufu_exp2(a1);
          ls2 = fadd2(ls2, f2_pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(lane_base + s_col + 32 * bb, pk);
      };
      // the first 64 keys' P; the MMA warp may start the P.V on those keys
      // while the rest of P is computed
      p_block(0);
      if (any_resc && n_pv > 0) {
        // O must be final before this tile's P.V starts (every earlier P.V
        // of this tile completed before S(j) did)
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(lane_base + o_col + 32 * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(lane_base + o_col + 32 * cc, o);
        }
      }
      send_first_half();
#pragma unroll
      for (int bb = 1; bb < BC / 64; ++bb) p_block(bb);
      float ls0, ls1;
      f2_unpack(ls2, ls0, ls1);
      float ls = ls0 + ls1;
      if (is_proxy) {
        // every summary stands for Bc keys except the final block's n_last
        ls = (float)BC * ls;
        if (x_last != -INFINITY) ls -= (float)(BC - p.n_last) * mufu_exp2(fmaf(x_last, c, -mref_s));
      }
      l = l * alpha + ls;
      m_true = m_new;
      m_ref = m_ref_new;
    } else {
      // the tile is skipped by this query tile; when the other half of a
      // 64-row pair keeps it, this half's P is zero
      if (keep_h[0] || keep_h[1]) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
#pragma unroll
        for (int h = 0; h < BC / 64; ++h) tmem_st32(lane_base + s_col + 32 * h, pk);
      }
      send_first_half();
    }
    const bool tile_keep = keep_h[0] || keep_h[1];
    const bool my_keep = mine;
    if (leader && my_vis) {
      if (!my_keep) {
        ++skipped;
        skip_word |= 1u << (j & 31);
        if (MASK && p.skip_bits != nullptr) {
          // steps walk the listed key tiles: record key tile kt itself
          const int qt = p.half ? 2 * pt + half : pt;
          atomicOr(p.skip_bits + ((size_t)(b * p.Hq + hq) * p.nQ + qt) * p.nKw + (kt >> 5), 1u << (kt & 31));
        }
      }
      if (DBG && p.skip_bits != nullptr && ((j & 31) == 31 || j == my_nvis - 1)) {
        const int qt = p.half ? 2 * pt + half : pt;
        p.skip_bits[((size_t)(b * p.Hq + hq) * p.nQ + qt) * p.nKw + (j >> 5)] = skip_word;
        skip_word = 0;
      }
    }
    // P (or nothing, for a skipped tile) is in TMEM: hand the step to the MMA warp
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready[t]));
    if (tile_keep) ++n_pv;
  }

  // ---- epilogue
  bool okf = true;
  if (nvis > 0) okf = mbar_wait(smem_u32(&bars->o_done[t]), 0, p.wait_ns);
  if (!okf) record_failure(p, bars);
  okf = __all_sync(0xffffffffu, okf) && !failed;
  tc_fence_after();
  const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
  __nv_bfloat16* orow = p.out + ((size_t)(b * p.Lq + grow) * p.Hq + hq) * D;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    if (okf && n_pv > 0) {
      tmem_ld32(lane_base + o_col + 32 * c, o);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0u;
    }
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
      for (int v8 = 0; v8 < 4; ++v8) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(o[8 * v8 + 0]) * inv_l, __uint_as_float(o[8 * v8 + 1]) * inv_l);
        w.y = pack_bf16x2(__uint_as_float(o[8 * v8 + 2]) * inv_l, __uint_as_float(o[8 * v8 + 3]) * inv_l);
        w.z = pack_bf16x2(__uint_as_float(o[8 * v8 + 4]) * inv_l, __uint_as_float(o[8 * v8 + 5]) * inv_l);
        w.w = pack_bf16x2(__uint_as_float(o[8 * v8 + 6]) * inv_l, __uint_as_float(o[8 * v8 + 7]) * inv_l);
        dst[v8] = w;
      }
    }
  }
  if (valid)
    p.lse[(size_t)(b * p.Hq + hq) * p.Lq + grow] = (l > 0.f) ? m_ref * p.scale + logf(l) : -INFINITY;
  if (leader) {
    const int qt = p.half ? 2 * pt + half : pt;
    if (qt < p.nQ) {
      if (p.skip_count != nullptr) p.skip_count[(size_t)(b * p.Hq + hq) * p.nQ + qt] = skipped;
      if (p.skip_bits != nullptr) {
        uint32_t* sb = p.skip_bits + ((size_t)(b * p.Hq + hq) * p.nQ + qt) * p.nKw;
        for (int w = (my_nvis + 31) / 32; w < p.nKw; ++w) sb[w] = 0u;
      }
    }
  }
}

template <int D, int BC, int NM_M, int VAR>
__global__ void __launch_bounds__(NTHREADS, 1)
    ssa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_km,
                   const __grid_constant__ CUtensorMap tm_vs, const Params p) {
  using L = Smem<D, BC>;
  constexpr int KST = L::KST, VST = L::VST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::BAR_OFF);
  const uint32_t q_s = smem_u32(smem + L::Q_OFF);
  const uint32_t k_s = smem_u32(smem + L::K_OFF);
  const uint32_t v_s = smem_u32(smem + L::V_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool skip_on = (p.mode & SSA_MODE_SKIP) != 0;
  // the MMA warp reads the softmax's per-step keep bytes whenever a tile may
  // be left out (skip-softmax, or key blocks selected by bitmap, where one
  // half of a 64-row pair may not select a key tile the other does); the V
  // producer reads them only with skip-softmax
  constexpr bool MASK = VAR >= 2, PROXY = VAR == 3;
  const bool vote_on = skip_on || MASK;

  // ---- work item.  Causal: heaviest pairs of query tiles first (the last
  // pair visits the most key tiles), query heads that share a KV head
  // adjacent.  Without a causal mask every pair costs the same: all pairs of
  // one query head are adjacent, so the CTAs running at one time read the K
  // and V of one or two heads, which stay in L2.
  Work wk;
  {
    const int per_pair = p.B * p.Hq;
    const int npairs = (p.nQp + 1) / 2;
    int pair, bh;
    if (p.causal) {
      pair = npairs - 1 - (int)(blockIdx.x / per_pair);
      bh = blockIdx.x % per_pair;
    } else {
      pair = blockIdx.x % npairs;
      bh = blockIdx.x / npairs;
    }
    wk.b = bh / p.Hq;
    wk.hq = bh % p.Hq;
    wk.hkv = wk.hq / (p.Hq / p.Hkv);
    wk.nvis = 0;
#pragma unroll
    for (int t = 0; t < NQT; ++t) {
      const int pt = 2 * pair + t;
      wk.pt[t] = pt;
      if (pt >= p.nQp) {
        wk.nvis_h[t][0] = wk.nvis_h[t][1] = 0;
      } else if (p.half) {
        wk.nvis_h[t][0] = (2 * pt < p.nQ) ? visited_key_tiles(p.causal, p.Lq, p.Lk, 64, BC, 2 * pt) : 0;
        wk.nvis_h[t][1] = (2 * pt + 1 < p.nQ) ? visited_key_tiles(p.causal, p.Lq, p.Lk, 64, BC, 2 * pt + 1) : 0;
      } else {
        wk.nvis_h[t][0] = wk.nvis_h[t][1] = visited_key_tiles(p.causal, p.Lq, p.Lk, BM, BC, pt);
      }
      wk.nvis_t[t] = wk.nvis_h[t][0] > wk.nvis_h[t][1] ? wk.nvis_h[t][0] : wk.nvis_h[t][1];
      if (wk.nvis_t[t] > wk.nvis) wk.nvis = wk.nvis_t[t];
    }
  }
  int nvis = wk.nvis;

  // ---- block-mask mode: the CTA walks the key tiles that any of its logical
  // query tiles selects and can see, in ascending order (warp 3 lists them
  // with, per step, which logical query tiles take part)
  if (MASK && warp == 3) {
    int last[4], qts[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int t = x >> 1, h = x & 1;
      last[x] = wk.nvis_h[t][h] - 1;  // last visible key tile (-1: none)
      qts[x] = p.half ? 2 * wk.pt[t] + h : wk.pt[t];
    }
    const int maxlast = max(max(last[0], last[1]), max(last[2], last[3]));
    int count = 0, end0 = 0, end1 = 0;
    for (int base = 0; base <= maxlast; base += 32) {
      const int kt = base + lane;
      uint32_t bits = 0;
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        if (kt <= last[x]) {
          const uint32_t w = p.block_mask[((size_t)(wk.b * p.Hkv + wk.hkv) * p.nQ + qts[x]) * p.nKw + (kt >> 5)];
          bits |= ((w >> (kt & 31)) & 1u) << x;
        }
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
      const int pos = count + __popc(bal & ((1u << lane) - 1u));
      if (bits != 0u && pos < MAX_LISTED_TILES) {
        bars->ktile[pos] = (uint16_t)kt;
        bars->part[pos] = (uint8_t)bits;
      }
      // one past each tile's last step so far: the listed lanes up to and
      // including the highest lane in which the tile takes part
      const uint32_t b0 = __ballot_sync(0xffffffffu, (bits & 3u) != 0u);
      const uint32_t b1 = __ballot_sync(0xffffffffu, (bits & 12u) != 0u);
      if (b0) end0 = count + __popc(bal & (0xffffffffu >> __clz(b0)));
      if (b1) end1 = count + __popc(bal & (0xffffffffu >> __clz(b1)));
      count += __popc(bal);
    }
    if (lane == 0) {
      bars->listed = min(count, MAX_LISTED_TILES);
      bars->listed_t[0] = min(end0, MAX_LISTED_TILES);
      bars->listed_t[1] = min(end1, MAX_LISTED_TILES);
    }
  }

  // ---- set-up
  if (tid == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < KST; ++i) {
      mbar_init(smem_u32(&bars->k_full[i]), 1);
      mbar_init(smem_u32(&bars->k_empty[i]), 1);
    }
    for (int i = 0; i < VST; ++i) {
      mbar_init(smem_u32(&bars->v_full[i]), 1);
      mbar_init(smem_u32(&bars->v_empty[i]), 1);
    }
    for (int i = 0; i < NQT; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      for (int v = 0; v < VSLOTS; ++v) mbar_init(smem_u32(&bars->vote_bar[i][v]), 4);
      mbar_init(smem_u32(&bars->p_ready[i]), 4);  // one arrival per softmax warp
      mbar_init(smem_u32(&bars->p_half[i]), 4);
      mbar_init(smem_u32(&bars->o_done[i]), 1);
    }
    mbar_init(smem_u32(&bars->mma_done), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (PROXY) {
      tma_prefetch_desc(&tm_km);
      tma_prefetch_desc(&tm_vs);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int listed = MASK ? bars->listed : 0;
  if (MASK) {
    wk.nvis_t[0] = bars->listed_t[0];
    wk.nvis_t[1] = bars->listed_t[1];
    nvis = wk.nvis = listed;
  }
  if (PROXY) {
    // no causal mask here: a query tile that exists visits every exact step,
    // then every proxy step
#pragma unroll
    for (int t = 0; t < NQT; ++t) {
      const bool exists = wk.nvis_h[t][0] > 0 || wk.nvis_h[t][1] > 0;
      wk.nvis_t[t] = exists ? listed + p.nP : 0;
    }
    nvis = wk.nvis = listed + p.nP;
  }
  // key tile (or, for a proxy step, summary chunk) of step j, and its maps
  auto key_tile = [&](int j) { return (PROXY && j >= listed) ? j - listed : MASK ? (int)bars->ktile[j] : j; };
  auto k_map = [&](int j) { return (PROXY && j >= listed) ? &tm_km : &tm_k; };
  auto v_map = [&](int j) { return (PROXY && j >= listed) ? &tm_vs : &tm_v; };
  // tile t takes part in step j: the first nvis_t[t] steps, or with key blocks
  // selected by bitmap the listed steps it selects (every proxy step when the
  // tile exists)
  auto part_of = [&](int t, int j) -> bool {
    if constexpr (!MASK) {
      return j < wk.nvis_t[t];
    } else {
      if (j >= wk.nvis_t[t]) return false;
      if (PROXY && j >= listed) return true;
      return ((bars->part[j] >> (2 * t)) & 3u) != 0u;
    }
  };

  if (warp < 4) {
    reg_dealloc<104>();
    if (warp == 0 && lane == 0 && nvis > 0) {
      // ======================= Q / K producer =======================
      const uint32_t qbar = smem_u32(&bars->q_full);
      uint32_t qbytes = 0;
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (wk.nvis_t[t] > 0) qbytes += L::QT_BYTES;
      mbar_arrive_expect_tx(qbar, qbytes);
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (wk.nvis_t[t] > 0)
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(q_s + t * L::QT_BYTES + c * BM * 128, &tm_q, qbar, c * 64, wk.hq, wk.pt[t] * BM, wk.b);
      int issued = 0;
      for (int j = 0; j < nvis; ++j) {
        const int slot = j % KST;
        if (aborted(bars)) break;
        if (!mbar_wait(smem_u32(&bars->k_empty[slot]), ((j / KST) & 1) ^ 1, p.wait_ns)) {
          record_failure(p, bars);
          break;
        }
        const uint32_t fb = smem_u32(&bars->k_full[slot]);
        mbar_arrive_expect_tx(fb, L::K_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(k_s + slot * L::K_BYTES + c * BC * 128, k_map(j), fb, c * 64, wk.hkv, key_tile(j) * BC, wk.b);
        issued = j + 1;
      }
      // drain: the newest load of each slot (older ones were consumed)
      bool drained = mbar_wait(qbar, 0, DRAIN_TIMEOUT_NS);
      for (int j = issued - KST; j < issued; ++j)
        if (j >= 0) drained &= mbar_wait(smem_u32(&bars->k_full[j % KST]), (j / KST) & 1, DRAIN_TIMEOUT_NS);
      if (!drained) record_failure(p, bars);
    } else if (warp == 2 && lane == 0) {
      // ======================= V producer =======================
      int last_load[VST];
      for (int i = 0; i < VST; ++i) last_load[i] = -1;
      int n_loads = 0;  // V tiles this CTA loaded (evidence output)
      int step_t[NQT] = {0, 0};  // steps each tile took part in so far
      for (int j = 0; j < nvis; ++j) {
        if (aborted(bars)) break;
        const int slot = j % VST;
        if (!mbar_wait(smem_u32(&bars->v_empty[slot]), ((j / VST) & 1) ^ 1, p.wait_ns)) {
          record_failure(p, bars);
          break;
        }
        const uint32_t fb = smem_u32(&bars->v_full[slot]);
        bool loaded = false, fail = false;
#pragma unroll
        for (int t = 0; t < NQT; ++t) {
          if (!part_of(t, j)) continue;
          bool keep = true;
          // Without skip-softmax a tile that takes part in a step keeps it (the
          // rows of a query tile that selects the key tile vote to keep), so V
          // is loaded at once; with it, only after the tile's votes are in.
          if (skip_on) {
            // the tile's own step count picks the vote slot and phase
            const int i = MASK ? step_t[t]++ : j;
            if (!mbar_wait_fast(smem_u32(&bars->vote_bar[t][i % VSLOTS]), (i / VSLOTS) & 1, p.wait_ns)) {
              fail = true;
              break;
            }
            keep = ld_shared_u32(smem_u32(&bars->vote[t][i % VSLOTS])) != 0u;
          }
          if (keep && !loaded) {
            mbar_arrive_expect_tx(fb, L::V_BYTES);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(v_s + slot * L::V_BYTES + c * BC * 128, v_map(j), fb, c * 64, wk.hkv, key_tile(j) * BC, wk.b);
            last_load[slot] = j;
            loaded = true;
            ++n_loads;
          }
        }
        if (fail) {
          record_failure(p, bars);
          break;
        }
        if (!loaded) {
          // the MMA warp released this slot's previous load before this use
          mbar_arrive(fb);
          last_load[slot] = -1;
        }
      }
      // drain: a load still owning its slot may be in flight only after a
      // failure; in the normal path this returns at once
      for (int i = 0; i < VST; ++i)
        if (last_load[i] >= 0 &&
            !mbar_wait(smem_u32(&bars->v_full[i]), (last_load[i] / VST) & 1, DRAIN_TIMEOUT_NS))
          record_failure(p, bars);
      if (p.v_loads != nullptr)
        p.v_loads[((size_t)wk.b * p.Hq + wk.hq) * ((p.nQp + 1) / 2) + wk.pt[0] / 2] = n_loads;
    } else if (warp == 1 && lane == 0 && nvis > 0) {
      // ======================= MMA issuer =======================
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BC, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, true);
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0, p.wait_ns);
      int k_ready = -1;  // newest K tile whose arrival was observed
      auto issue_qk = [&](int t, int j) -> bool {
        const int slot = j % KST;
        if (k_ready < j) {
          if (!mbar_wait_fast(smem_u32(&bars->k_full[slot]), (j / KST) & 1, p.wait_ns)) return false;
          k_ready = j;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + 256 * t;
        const uint32_t qt_s = q_s + t * L::QT_BYTES;
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t off = (s >> 2) * (BM * 128) + (s & 3) * 32;
          const uint32_t koff = (s >> 2) * (BC * 128) + (s & 3) * 32;
          const uint64_t ad = smem_desc_sw128(qt_s + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_s + slot * L::K_BYTES + koff, 16, 1024);
          mma_ss(d_tmem, ad, bd, idesc_qk, s > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars->s_full[t]));
        return true;
      };
      // last tile that reads K tile j: B when it takes part in step j, else A
      auto k_last_user = [&](int j) { return part_of(1, j) ? 1 : 0; };
      int pv_count[NQT] = {0, 0};
      int step_t[NQT] = {0, 0};  // steps each tile took part in so far
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (ok && part_of(t, 0)) {
          ok = issue_qk(t, 0);
          if (ok && k_last_user(0) == t) mma_commit(smem_u32(&bars->k_empty[0]));
        }
      for (int j = 0; ok && j < nvis; ++j) {
        if (aborted(bars)) { ok = false; break; }
        const int slot = j % VST;
        bool v_seen = false, any_pv = false;
#pragma unroll
        for (int t = 0; t < NQT; ++t) {
          // a tile's next QK^T is issued while walking the step before it, so
          // that it never waits on a K tile whose slot a later step frees
          const bool next = j + 1 < nvis && part_of(t, j + 1);
          if (!part_of(t, j)) {
            if constexpr (MASK) {
              if (next) {
                if (!issue_qk(t, j + 1)) { ok = false; break; }
                if (k_last_user(j + 1) == t) mma_commit(smem_u32(&bars->k_empty[(j + 1) % KST]));
              }
            }
            continue;
          }
          // the tile's own step: barrier phases and vote slot (without a
          // bitmap a tile takes part in a prefix of the steps)
          const int i = MASK ? step_t[t]++ : j;
          // P.V in two parts: the first 64 keys once their P is in TMEM, the
          // rest when the whole of P is
          if (!mbar_wait_fast(smem_u32(&bars->p_half[t]), i & 1, p.wait_ns)) { ok = false; break; }
          const bool keep = !vote_on || ld_shared_u32(smem_u32(&bars->vote[t][i % VSLOTS])) != 0u;
          const uint32_t p_tmem = tmem + 256 * t;
          auto issue_pv = [&](int k0, int k1) {
            tc_fence_after();
#pragma unroll
            for (int s = k0; s < k1; ++s) {
              const uint64_t bd = smem_desc_sw128(v_s + slot * L::V_BYTES + s * 16 * 128, BC * 128, 1024);
              mma_ts(tmem + 256 * t + 128, p_tmem + s * 8, bd, idesc_pv, (pv_count[t] > 0 || s > 0) ? 1u : 0u);
            }
          };
          if (keep) {
            if (!v_seen) {
              if (!mbar_wait_fast(smem_u32(&bars->v_full[slot]), (j / VST) & 1, p.wait_ns)) { ok = false; break; }
              v_seen = true;
            }
            issue_pv(0, 4);
          }
          if (!mbar_wait_fast(smem_u32(&bars->p_ready[t]), i & 1, p.wait_ns)) { ok = false; break; }
          if (keep) {
            issue_pv(4, BC / 16);
            ++pv_count[t];
            any_pv = true;
          }
          if (j == wk.nvis_t[t] - 1) mma_commit(smem_u32(&bars->o_done[t]));
          if (next) {
            if (!issue_qk(t, j + 1)) { ok = false; break; }
            if (k_last_user(j + 1) == t) mma_commit(smem_u32(&bars->k_empty[(j + 1) % KST]));
          }
        }
        if (!ok) break;
        if (!v_seen && !mbar_wait_fast(smem_u32(&bars->v_full[slot]), (j / VST) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        if (any_pv) mma_commit(smem_u32(&bars->v_empty[slot]));
        else mbar_arrive(smem_u32(&bars->v_empty[slot]));
      }
      if (!ok) {
        record_failure(p, bars);
        // unblock the softmax epilogues (they see the failure flag)
        mma_commit(smem_u32(&bars->o_done[0]));
        mma_commit(smem_u32(&bars->o_done[1]));
      }
      // every MMA this thread issued has completed before TMEM is freed
      mma_commit(smem_u32(&bars->mma_done));
      if (!mbar_wait(smem_u32(&bars->mma_done), 0, DRAIN_TIMEOUT_NS)) record_failure(p, bars);
    }
  } else {
    reg_alloc<200>();
    const int t = warp >> 3;  // warps 4-7: tile A, 8-11: tile B
    softmax_tile<D, BC, NM_M, VAR>(p, bars, wk.b, wk.hq, wk.hkv, t, t ? wk.pt[1] : wk.pt[0],
                                   t ? wk.nvis_h[1][0] : wk.nvis_h[0][0],
                                   t ? wk.nvis_h[1][1] : wk.nvis_h[0][1],
                                   t ? wk.nvis_t[1] : wk.nvis_t[0], tmem);
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ============================================================ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static std::mutex g_mu;
static unsigned long long g_wait_ns = WAIT_TIMEOUT_NS;
static EncodeTiledFn g_encode = nullptr;
constexpr int MAX_DEV = 64;
static int* g_status[MAX_DEV] = {};
static bool g_attr_set[MAX_DEV][80] = {};

static EncodeTiledFn encode_fn() {
  if (g_encode) return g_encode;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return g_encode;
}

// [B, L, H, d] bf16 -> 4-D map (d, H, L, B), box (64, 1, rows, 1), 128B swizzle,
// zero fill outside the tensor (ragged tails read zeros).
static bool make_map(CUtensorMap* map, const void* base, int B, int L, int H, int d, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)L * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int* status_word(int dev) {
  if (dev < 0 || dev >= MAX_DEV) return nullptr;
  if (!g_status[dev]) {
    int* w = nullptr;
    if (cudaMalloc(&w, sizeof(int)) != cudaSuccess) return nullptr;
    if (cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return nullptr;
    g_status[dev] = w;
  }
  return g_status[dev];
}

bool tma_map_bf16(CUtensorMap* map, const void* base, int B, int L, int H, int d, int rows) {
  std::lock_guard<std::mutex> g(g_mu);
  return make_map(map, base, B, L, H, d, rows);
}

int* device_status_word(int dev) {
  std::lock_guard<std::mutex> g(g_mu);
  return status_word(dev);
}

unsigned long long wait_timeout_ns() {
  std::lock_guard<std::mutex> g(g_mu);
  return g_wait_ns;
}

struct Maps {
  CUtensorMap q, k, v, km, vs;  // km / vs: proxy summaries (copies of k / v when unused)
};

template <int D, int BC, int NM_M, int VAR>
static int launch_one(const Maps& mp, const Params& p, int grid, cudaStream_t stream, int dev, int inst) {
  using L = Smem<D, BC>;
  if (!g_attr_set[dev][inst]) {
    if (cudaFuncSetAttribute(ssa_fwd_kernel<D, BC, NM_M, VAR>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC) != cudaSuccess)
      return SSA_ERR_CUDA;
    g_attr_set[dev][inst] = true;
  }
  ssa_fwd_kernel<D, BC, NM_M, VAR><<<grid, NTHREADS, L::ALLOC, stream>>>(mp.q, mp.k, mp.v, mp.km, mp.vs, p);
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

// One instance per (N:M group width or none) x (plain, debug outputs, key
// blocks by bitmap), so the plain skip-softmax kernel carries no N:M, debug or
// bitmap code; proxy compensation (no N:M) has one instance per shape.
template <int D, int BC, int NM_M>
static int launch_var(const Maps& mp, const Params& p, int grid, cudaStream_t stream, int dev, int inst) {
  if (p.block_mask != nullptr) return launch_one<D, BC, NM_M, 2>(mp, p, grid, stream, dev, inst + 2);
  if (p.skip_bits != nullptr || p.keep_bits != nullptr || p.v_loads != nullptr)
    return launch_one<D, BC, NM_M, 1>(mp, p, grid, stream, dev, inst + 1);
  return launch_one<D, BC, NM_M, 0>(mp, p, grid, stream, dev, inst);
}

template <int D, int BC>
static int launch(const Maps& mp, const Params& p, int grid, cudaStream_t stream, int dev, int base) {
  constexpr int PER = 18;  // instances per shape: 6 N:M codes x 3 variants
  if (p.nP > 0) return launch_one<D, BC, 0, 3>(mp, p, grid, stream, dev, 4 * PER + base);
  // N = M keeps every key: the instance without N:M computes exactly that
  const int nm = ((p.mode & SSA_MODE_NM) && p.n < p.m) ? p.m : 0;
  // 0 none, 1 eight-wide, 2..4 four-wide N = 1..3, 5 eight-wide N = 4
  const int code = nm == 0 ? 0 : nm == 8 ? (p.n == 4 ? 5 : 1) : 1 + p.n;
  const int inst = base * PER + 3 * code;
  switch (code) {
    case 0: return launch_var<D, BC, 0>(mp, p, grid, stream, dev, inst);
    case 1: return launch_var<D, BC, 8>(mp, p, grid, stream, dev, inst);
    case 2: return launch_var<D, BC, 41>(mp, p, grid, stream, dev, inst);
    case 3: return launch_var<D, BC, 42>(mp, p, grid, stream, dev, inst);
    case 4: return launch_var<D, BC, 43>(mp, p, grid, stream, dev, inst);
    default: return launch_var<D, BC, 84>(mp, p, grid, stream, dev, inst);
  }
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
static bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

static int run(const void* q, const void* k, const void* v, void* out, float* lse,
               int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
               float scale, int mode, float lambda, int n, int m, int sink, int recent, int Br,
               int Bc, void* stream, uint32_t* skip_bits, uint32_t* keep_bits,
               int* status_override = nullptr, const uint32_t* block_mask = nullptr,
               int32_t* v_loads = nullptr, const void* kmean = nullptr, const void* vsum = nullptr) {
  // ---- argument checks (synchronous, nothing launched on failure)
  const bool proxy = kmean != nullptr || vsum != nullptr;
  if (!q || !k || !v || !out || !lse || (!tile_skip_count && !proxy)) return SSA_ERR_INVALID_ARG;
  if (proxy && (!kmean || !vsum || !block_mask || !aligned16(kmean) || !aligned16(vsum)))
    return SSA_ERR_INVALID_ARG;
  if (proxy && (causal || mode != SSA_MODE_DENSE)) return SSA_ERR_UNSUPPORTED;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Lk <= 0 || d <= 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (mode < 0 || mode > 3) return SSA_ERR_INVALID_ARG;
  if ((mode & SSA_MODE_SKIP) && (!std::isfinite(lambda) || lambda < 0.f)) return SSA_ERR_INVALID_ARG;
  if ((mode & SSA_MODE_NM) && (sink < 0 || recent < 0)) return SSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return SSA_ERR_INVALID_ARG;
  // 32-bit outputs: a misaligned one would fault in the kernel
  if (!aligned4(tile_skip_count) || !aligned4(skip_bits) || !aligned4(keep_bits) || !aligned4(v_loads))
    return SSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSA_ERR_UNSUPPORTED;
  if ((Br != 64 && Br != 128) || (Bc != 64 && Bc != 128)) return SSA_ERR_UNSUPPORTED;
  if (mode & SSA_MODE_NM) {
    if (!((m == 4 && n >= 1 && n <= 4) || (m == 8 && n >= 1 && n <= 8))) return SSA_ERR_UNSUPPORTED;
    if (Bc % m != 0) return SSA_ERR_UNSUPPORTED;
  }
  if (block_mask != nullptr) {
    if ((reinterpret_cast<uintptr_t>(block_mask) & 3u) != 0u) return SSA_ERR_INVALID_ARG;
    if ((Lk + Bc - 1) / Bc > MAX_LISTED_TILES) return SSA_ERR_UNSUPPORTED;
  }
  const long long nQp = (Lq + BM - 1) / BM;
  const long long grid = ((nQp + 1) / 2) * B * Hq;
  if (grid > 0x7fffffffLL) return SSA_ERR_UNSUPPORTED;
  if ((long long)B * Lq * Hq * d >= (1LL << 40) || (long long)B * Lk * Hkv * d >= (1LL << 40))
    return SSA_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return SSA_ERR_CUDA;
  Maps mp;
  Params p{};
  const int nK = (Lk + Bc - 1) / Bc;
  {
    std::lock_guard<std::mutex> g(g_mu);
    p.status = status_override ? status_override : status_word(dev);
    if (!p.status) return SSA_ERR_CUDA;
    if (!make_map(&mp.q, q, B, Lq, Hq, d, BM) || !make_map(&mp.k, k, B, Lk, Hkv, d, Bc) ||
        !make_map(&mp.v, v, B, Lk, Hkv, d, Bc))
      return SSA_ERR_CUDA;
    if (proxy) {
      // summaries [B, nK, Hkv, d]: one row per key block, loaded Bc rows at a time
      if (!make_map(&mp.km, kmean, B, nK, Hkv, d, Bc) || !make_map(&mp.vs, vsum, B, nK, Hkv, d, Bc))
        return SSA_ERR_CUDA;
    } else {
      mp.km = mp.k;
      mp.vs = mp.v;
    }
  }
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.skip_count = tile_skip_count;
  p.skip_bits = skip_bits;
  p.keep_bits = keep_bits;
  p.v_loads = v_loads;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk; p.causal = causal ? 1 : 0;
  p.mode = mode;
  p.n = (mode & SSA_MODE_NM) ? n : 0;
  p.m = (mode & SSA_MODE_NM) ? m : 4;
  p.sink = (mode & SSA_MODE_NM) ? sink : 0;
  p.recent = (mode & SSA_MODE_NM) ? recent : 0;
  p.half = (Br == 64) ? 1 : 0;
  p.nQp = (int)nQp;
  p.nQ = (Lq + Br - 1) / Br;
  p.nK = (Lk + Bc - 1) / Bc;
  p.nKw = (p.nK + 31) / 32;
  p.Lkw = (Lk + 31) / 32;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.log2_lambda = ((mode & SSA_MODE_SKIP) && lambda > 0.f) ? (float)std::log2((double)lambda)
                                                           : -INFINITY;
  p.wait_ns = g_wait_ns;
  p.block_mask = block_mask;
  p.nP = proxy ? (nK + Bc - 1) / Bc : 0;
  p.n_last = Lk - (nK - 1) * Bc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // A caller-supplied status word (the allocation-free entry point's shared
  // scratch) keeps the previous call's contents: clear it on the stream first.
  if (status_override && cudaMemsetAsync(status_override, 0, sizeof(int), st) != cudaSuccess)
    return SSA_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_mu);
  if (d == 128 && Bc == 128) return launch<128, 128>(mp, p, (int)grid, st, dev, 0);
  if (d == 128 && Bc == 64) return launch<128, 64>(mp, p, (int)grid, st, dev, 1);
  if (d == 64 && Bc == 128) return launch<64, 128>(mp, p, (int)grid, st, dev, 2);
  return launch<64, 64>(mp, p, (int)grid, st, dev, 3);
}


// ------------------------------------------------------------------------
// Allocation-free variant.  Its only scratch is the kernel's status word (the
// flag a CTA raises when one of its bounded waits times out); here it lives in
// this file-scope device array instead of a lazily cudaMalloc'd word.  Every
// GPU that loads the library holds the array until the process exits.
constexpr int NOALLOC_SCRATCH_BYTES = 256;
static __device__ __align__(256) int g_noalloc_scratch[NOALLOC_SCRATCH_BYTES / sizeof(int)];
static int* g_noalloc_addr[MAX_DEV] = {};

// Scratch one call needs: the 4-byte status word, whatever the problem size.
static size_t noalloc_scratch_bytes() { return sizeof(int); }

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with that device current.
static int* noalloc_scratch(int dev) {
  if (dev < 0 || dev >= MAX_DEV) return nullptr;
  if (!g_noalloc_addr[dev]) {
    int* ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch) != cudaSuccess)
      return nullptr;
    g_noalloc_addr[dev] = ptr;
  }
  return g_noalloc_addr[dev];
}

static int run_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                       int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                       int causal, float scale, int mode, float lambda, int n, int m, int sink,
                       int recent, int Br, int Bc, void* stream) {
  if (noalloc_scratch_bytes() > (size_t)NOALLOC_SCRATCH_BYTES) return SSA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return SSA_ERR_CUDA;
  int* scratch;
  {
    std::lock_guard<std::mutex> g(g_mu);
    scratch = noalloc_scratch(dev);
  }
  if (!scratch) return SSA_ERR_CUDA;
  return run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode, lambda,
             n, m, sink, recent, Br, Bc, stream, nullptr, nullptr, scratch);
}

}  // namespace ssa

extern "C" {

int ssa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
            int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
            float scale, int mode, float lambda, int n, int m, int sink, int recent, int Br, int Bc,
            void* stream) {
  return ssa::run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                  lambda, n, m, sink, recent, Br, Bc, stream, nullptr, nullptr);
}

int ssa_fwd_debug(const void* q, const void* k, const void* v, void* out, float* lse,
                  int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                  int causal, float scale, int mode, float lambda, int n, int m, int sink,
                  int recent, int Br, int Bc, void* stream, uint32_t* skip_bits,
                  uint32_t* keep_bits, int32_t* v_tile_loads) {
  return ssa::run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                  lambda, n, m, sink, recent, Br, Bc, stream, skip_bits, keep_bits, nullptr, nullptr,
                  v_tile_loads);
}

int ssa_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                    int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                    int causal, float scale, int mode, float lambda, int n, int m, int sink,
                    int recent, int Br, int Bc, void* stream) {
  return ssa::run_noalloc(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale,
                          mode, lambda, n, m, sink, recent, Br, Bc, stream);
}

int ssa_fwd_blockmask(const void* q, const void* k, const void* v, void* out, float* lse,
                      int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                      int causal, float scale, int mode, float lambda, int n, int m, int sink,
                      int recent, int Br, int Bc, const uint32_t* block_mask, void* stream) {
  if (!block_mask) return SSA_ERR_INVALID_ARG;
  return ssa::run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                  lambda, n, m, sink, recent, Br, Bc, stream, nullptr, nullptr, nullptr, block_mask);
}

int ssa_fwd_blockmask_debug(const void* q, const void* k, const void* v, void* out, float* lse,
                            int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                            int causal, float scale, int mode, float lambda, int n, int m, int sink,
                            int recent, int Br, int Bc, const uint32_t* block_mask, void* stream,
                            uint32_t* skip_bits, int32_t* v_tile_loads) {
  if (!block_mask) return SSA_ERR_INVALID_ARG;
  return ssa::run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                  lambda, n, m, sink, recent, Br, Bc, stream, skip_bits, nullptr, nullptr, block_mask,
                  v_tile_loads);
}

int ssa_fwd_blockmask_proxy(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                            int Hq, int Hkv, int Lq, int Lk, int d, float scale, int Br, int Bc,
                            const uint32_t* block_mask, const void* kmean, const void* vsum,
                            void* stream) {
  if (!block_mask || !kmean || !vsum) return SSA_ERR_INVALID_ARG;
  return ssa::run(q, k, v, out, lse, nullptr, B, Hq, Hkv, Lq, Lk, d, 0, scale, SSA_MODE_DENSE, 0.f, 0, 0,
                  0, 0, Br, Bc, stream, nullptr, nullptr, nullptr, block_mask, nullptr, kmean, vsum);
}

int64_t ssa_visited_tiles(int causal, int Lq, int Lk, int Br, int Bc) {
  if (Lq <= 0 || Lk <= 0 || Br <= 0 || Bc <= 0) return -1;
  const int nQ = (Lq + Br - 1) / Br;
  int64_t t = 0;
  for (int qt = 0; qt < nQ; ++qt) t += ssa::visited_key_tiles(causal, Lq, Lk, Br, Bc, qt);
  return t;
}

void ssa_set_wait_timeout_ns(uint64_t ns) {
  std::lock_guard<std::mutex> g(ssa::g_mu);
  ssa::g_wait_ns = ns ? (unsigned long long)ns : ssa::WAIT_TIMEOUT_NS;
}

int ssa_device_status(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SSA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= ssa::MAX_DEV) return SSA_ERR_CUDA;
  // The two words a timed-out wait can raise on this device: the one the
  // allocating entry points created (if any has run here) and the static one
  // of the allocation-free entry point (if it has run here).  Nothing is
  // allocated: a word that does not exist yet has recorded nothing.
  int* words[2];
  {
    std::lock_guard<std::mutex> g(ssa::g_mu);
    words[0] = ssa::g_status[dev];
    words[1] = ssa::g_noalloc_addr[dev];
  }
  bool timed_out = false;
  for (int* w : words) {
    if (!w) continue;
    int h = 0;
    if (cudaMemcpy(&h, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SSA_ERR_CUDA;
    if (h != 0) {
      if (cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return SSA_ERR_CUDA;
      timed_out = true;
    }
  }
  return timed_out ? SSA_ERR_TIMEOUT : SSA_OK;
}

const char* ssa_status_string(int status) {
  switch (status) {
    case SSA_OK: return "SSA_OK";
    case SSA_ERR_INVALID_ARG: return "SSA_ERR_INVALID_ARG";
    case SSA_ERR_UNSUPPORTED: return "SSA_ERR_UNSUPPORTED";
    case SSA_ERR_CUDA: return "SSA_ERR_CUDA";
    case SSA_ERR_TIMEOUT: return "SSA_ERR_TIMEOUT";
    default: return "SSA_ERR_UNKNOWN";
  }
}

int ssa_version(void) { return 100; }

}  // extern "C"
