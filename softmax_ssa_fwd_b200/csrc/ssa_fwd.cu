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
// One CTA owns 128 query rows of one (batch, query head) and walks the key
// tiles it can see.  Warp roles (256 threads):
//   warp 0      Q and K producer: TMA into a KST-deep K ring
//   warp 1      TMEM owner and MMA issuer: S = Q K^T and O += P V on tcgen05
//   warp 2      V producer: issues a V tile's TMA only after the tile's keep
//               decision, so a skipped tile never loads V
//   warps 4..7  softmax: thread t owns query row t (TMEM lane t); masks, N:M
//               top-N in registers, tile row max, skip vote, exp2, P -> TMEM,
//               lazy O rescale, epilogue
// TMEM (512 columns): S/P double buffer at columns 0 and 128, O at 256.
// P (bf16, two per 32-bit column) overwrites the S buffer it came from and is
// the A operand of the P.V MMA straight from TMEM.
//
// When Br = 64 the 128-row CTA tile carries two logical query tiles (rows
// 0-63 and 64-127) that vote, count and keep state separately; a V tile is
// loaded and P.V issued when either keeps the key tile, with P = 0 for the
// half that skipped.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/ssa.h"
#include "ptx.cuh"

namespace ssa {

constexpr int BM = 128;       // CTA query rows = tcgen05 M
constexpr int KST = 3;        // K ring depth
constexpr int VST = 2;        // V ring depth
constexpr int NTHREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr int S_COL = 0;      // S/P buffer b at column S_COL + 128 * b
constexpr int O_COL = 256;
constexpr uint64_t WAIT_TIMEOUT_NS = 2000000000ull;  // 2 s per wait
constexpr float RESCALE_LOG2 = 8.0f;  // lazy O rescale once the max grew by 2^8

struct Params {
  __nv_bfloat16* out;
  float* lse;
  int32_t* skip_count;
  uint32_t* skip_bits;  // optional
  uint32_t* keep_bits;  // optional
  int* status;
  int B, Hq, Hkv, Lq, Lk, causal, mode, n, m, sink, recent;
  int half;   // Br == 64
  int Br;
  int nQp;    // 128-row CTA tiles per (b, hq)
  int nQ;     // logical query tiles per (b, hq)
  int nK;     // key tiles
  int nKw;    // words of skip bits per logical query tile
  int Lkw;    // words of keep bits per row
  float scale;
  float scale_log2;
  float log2_lambda;  // -inf for lambda == 0
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[2], dec_ready[2], p_ready[2];
  uint64_t o_bar, o_final;
  uint32_t tmem_base;
  uint32_t dec_word[2];
  uint32_t vote[2][4];
  uint32_t abort_flag;
};

template <int D, int BC>
struct Smem {
  static constexpr uint32_t Q_BYTES = BM * D * 2;
  static constexpr uint32_t K_BYTES = BC * D * 2;
  static constexpr uint32_t V_BYTES = BC * D * 2;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + Q_BYTES;
  static constexpr uint32_t V_OFF = K_OFF + KST * K_BYTES;
  static constexpr uint32_t BAR_OFF = V_OFF + VST * V_BYTES;
  static constexpr uint32_t TOTAL = BAR_OFF + ((sizeof(Bars) + 127) / 128) * 128;
  static constexpr uint32_t ALLOC = TOTAL + 1024;  // slack for 1024-byte alignment
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

__device__ __forceinline__ float fast_exp2(float x) {
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

// N:M selection on one thread's row: for each aligned group of M keys keep a
// key iff it is visible and (inside the sink / recent window, or among the N
// largest scores of its group, equal scores ranked by lower index).  Dropped
// keys become -inf.  Returns a bit per column of the BC-wide tile.
template <int M, int BC>
__device__ __forceinline__ void nm_select(float (&x)[BC], int N, int col0, int pos, int sink,
                                          int recent) {
#pragma unroll
  for (int g = 0; g < BC / M; ++g) {
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
      const int jj = col0 + g * M + a;
      const int dist = pos - jj;
      const bool win = (jj < sink) || (dist >= 0 && dist < recent);
      if (!(win || rank[a] < N)) x[g * M + a] = -INFINITY;
    }
  }
}

template <int D, int BC>
__global__ void __launch_bounds__(NTHREADS, 1)
    ssa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using L = Smem<D, BC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::BAR_OFF);
  const uint32_t q_s = smem_u32(smem + L::Q_OFF);
  const uint32_t k_s = smem_u32(smem + L::K_OFF);
  const uint32_t v_s = smem_u32(smem + L::V_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item: heaviest causal tiles first; query heads that share a KV
  // head are adjacent in launch order.
  const int per_tile = p.B * p.Hq;
  int pt = blockIdx.x / per_tile;
  if (p.causal) pt = p.nQp - 1 - pt;
  const int bh = blockIdx.x % per_tile;
  const int b = bh / p.Hq, hq = bh % p.Hq;
  const int hkv = hq / (p.Hq / p.Hkv);

  int nvis_h[2];
  if (p.half) {
    nvis_h[0] = (2 * pt < p.nQ) ? visited_key_tiles(p.causal, p.Lq, p.Lk, 64, BC, 2 * pt) : 0;
    nvis_h[1] = (2 * pt + 1 < p.nQ) ? visited_key_tiles(p.causal, p.Lq, p.Lk, 64, BC, 2 * pt + 1) : 0;
  } else {
    nvis_h[0] = nvis_h[1] = visited_key_tiles(p.causal, p.Lq, p.Lk, BM, BC, pt);
  }
  const int nvis = nvis_h[0] > nvis_h[1] ? nvis_h[0] : nvis_h[1];

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
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->dec_ready[i]), 1);
      mbar_init(smem_u32(&bars->p_ready[i]), 1);
    }
    mbar_init(smem_u32(&bars->o_bar), 1);
    mbar_init(smem_u32(&bars->o_final), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ======================= Q / K producer =======================
    if (lane == 0 && nvis > 0) {
      const uint32_t qbar = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qbar, L::Q_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_4d(q_s + c * BM * 128, &tm_q, qbar, c * 64, hq, pt * BM, b);
      int issued = 0;
      for (int j = 0; j < nvis; ++j) {
        const int slot = j % KST;
        if (aborted(bars)) break;
        if (!mbar_wait(smem_u32(&bars->k_empty[slot]), ((j / KST) & 1) ^ 1, WAIT_TIMEOUT_NS)) {
          record_failure(p, bars);
          break;
        }
        const uint32_t fb = smem_u32(&bars->k_full[slot]);
        mbar_arrive_expect_tx(fb, L::K_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(k_s + slot * L::K_BYTES + c * BC * 128, &tm_k, fb, c * 64, hkv, j * BC, b);
        issued = j + 1;
      }
      // drain: the newest load of each slot (older ones were consumed)
      mbar_wait(qbar, 0, WAIT_TIMEOUT_NS);
      for (int j = issued - KST; j < issued; ++j)
        if (j >= 0) mbar_wait(smem_u32(&bars->k_full[j % KST]), (j / KST) & 1, WAIT_TIMEOUT_NS);
    }
  } else if (warp == 2) {
    // ======================= V producer =======================
    if (lane == 0) {
      int last_load[VST];
      for (int i = 0; i < VST; ++i) last_load[i] = -1;
      for (int j = 0; j < nvis; ++j) {
        if (aborted(bars)) break;
        if (!mbar_wait(smem_u32(&bars->dec_ready[j & 1]), (j >> 1) & 1, WAIT_TIMEOUT_NS)) {
          record_failure(p, bars);
          break;
        }
        const uint32_t keep = *reinterpret_cast<volatile uint32_t*>(&bars->dec_word[j & 1]);
        const int slot = j % VST;
        if (!mbar_wait(smem_u32(&bars->v_empty[slot]), ((j / VST) & 1) ^ 1, WAIT_TIMEOUT_NS)) {
          record_failure(p, bars);
          break;
        }
        const uint32_t fb = smem_u32(&bars->v_full[slot]);
        if (keep) {
          mbar_arrive_expect_tx(fb, L::V_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(v_s + slot * L::V_BYTES + c * BC * 128, &tm_v, fb, c * 64, hkv, j * BC, b);
          last_load[slot] = j;
        } else {
          mbar_arrive(fb);
        }
      }
      for (int i = 0; i < VST; ++i)
        if (last_load[i] >= 0)
          mbar_wait(smem_u32(&bars->v_full[i]), (last_load[i] / VST) & 1, WAIT_TIMEOUT_NS);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0 && nvis > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BC, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, true);
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0, WAIT_TIMEOUT_NS);
      auto issue_qk = [&](int j) -> bool {
        const int slot = j % KST;
        if (!mbar_wait(smem_u32(&bars->k_full[slot]), (j / KST) & 1, WAIT_TIMEOUT_NS)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + S_COL + 128 * (j & 1);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t off = (s >> 2) * (BM * 128) + (s & 3) * 32;
          const uint32_t koff = (s >> 2) * (BC * 128) + (s & 3) * 32;
          const uint64_t ad = smem_desc_sw128(q_s + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_s + slot * L::K_BYTES + koff, 16, 1024);
          mma_ss(d_tmem, ad, bd, idesc_qk, s > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars->k_empty[slot]));
        mma_commit(smem_u32(&bars->s_full[j & 1]));
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && nvis > 1) ok = issue_qk(1);
      int pv_count = 0;
      for (int j = 0; ok && j < nvis; ++j) {
        if (aborted(bars)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&bars->p_ready[j & 1]), (j >> 1) & 1, WAIT_TIMEOUT_NS)) { ok = false; break; }
        const uint32_t keep = *reinterpret_cast<volatile uint32_t*>(&bars->dec_word[j & 1]);
        const int slot = j % VST;
        if (!mbar_wait(smem_u32(&bars->v_full[slot]), (j / VST) & 1, WAIT_TIMEOUT_NS)) { ok = false; break; }
        tc_fence_after();
        if (keep) {
          const uint32_t p_tmem = tmem + S_COL + 128 * (j & 1);
#pragma unroll
          for (int s = 0; s < BC / 16; ++s) {
            const uint64_t bd =
                smem_desc_sw128(v_s + slot * L::V_BYTES + s * 16 * 128, BC * 128, 1024);
            mma_ts(tmem + O_COL, p_tmem + s * 8, bd, idesc_pv, (pv_count > 0 || s > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&bars->v_empty[slot]));
          mma_commit(smem_u32(&bars->o_bar));
          ++pv_count;
        } else {
          mbar_arrive(smem_u32(&bars->v_empty[slot]));
        }
        if (j + 2 < nvis && !issue_qk(j + 2)) { ok = false; break; }
      }
      if (!ok) record_failure(p, bars);
      mma_commit(smem_u32(&bars->o_final));
      mbar_wait(smem_u32(&bars->o_final), 0, WAIT_TIMEOUT_NS);
    }
  } else if (warp >= 4) {
    // ======================= softmax / epilogue =======================
    const int row = tid - 128;
    const int quarter = warp - 4;
    const int half = p.half ? (row >> 6) : 0;
    const int grow = pt * BM + row;
    const bool valid = grow < p.Lq;
    const int pos = grow + p.Lk - p.Lq;
    const int pos_first = pt * BM + p.Lk - p.Lq;  // position of the CTA's first row
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
    const bool skip_on = (p.mode & SSA_MODE_SKIP) != 0;
    const bool nm_on = (p.mode & SSA_MODE_NM) != 0;
    const bool leader = p.half ? ((row & 63) == 0) : (row == 0);
    const int my_nvis = nvis_h[half];

    float m_true = -INFINITY;  // running max over kept tiles (raw q.k units)
    float m_ref = -INFINITY;   // reference the O accumulator and l are scaled to
    float l = 0.f;
    int n_pv = 0;
    int skipped = 0;
    uint32_t skip_word = 0;
    bool failed = false;

    for (int j = 0; j < nvis; ++j) {
      bool ok = !failed && mbar_wait(smem_u32(&bars->s_full[j & 1]), (j >> 1) & 1, WAIT_TIMEOUT_NS);
      ok = __all_sync(0xffffffffu, ok);
      float x[BC];
      float m_tile = -INFINITY;
      const int col0 = j * BC;
      if (ok) {
        tc_fence_after();
        uint32_t sr[BC];
#pragma unroll
        for (int c = 0; c < BC / 32; ++c)
          tmem_ld32(lane_base + S_COL + 128 * (j & 1) + 32 * c,
                    *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < BC; ++i) x[i] = __uint_as_float(sr[i]);
        const bool need_mask = (col0 + BC > p.Lk) || (p.causal && col0 + BC - 1 > pos_first);
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < BC; ++i) {
            const int jj = col0 + i;
            if (jj >= p.Lk || (p.causal && jj > pos)) x[i] = -INFINITY;
          }
        }
        if (nm_on) {
          if (p.m == 4) nm_select<4, BC>(x, p.n, col0, pos, p.sink, p.recent);
          else nm_select<8, BC>(x, p.n, col0, pos, p.sink, p.recent);
        }
#pragma unroll
        for (int i = 0; i < BC; ++i) m_tile = fmaxf(m_tile, x[i]);
        if (p.keep_bits != nullptr && valid && j < my_nvis) {
          uint32_t* kb = p.keep_bits + ((size_t)(b * p.Hq + hq) * p.Lq + grow) * p.Lkw;
#pragma unroll
          for (int w = 0; w < BC / 32; ++w) {
            uint32_t word = 0;
#pragma unroll
            for (int t = 0; t < 32; ++t) word |= (x[32 * w + t] != -INFINITY ? 1u : 0u) << t;
            const int wi = col0 / 32 + w;
            if (wi < p.Lkw) kb[wi] = word;
          }
        }
      }
      const bool negligible =
          !valid || m_tile == -INFINITY ||
          (m_true != -INFINITY && (m_tile - m_true) * p.scale_log2 < p.log2_lambda);
      const uint32_t wneg = __all_sync(0xffffffffu, negligible) ? 1u : 0u;
      if (lane == 0) bars->vote[j & 1][quarter] = wneg | (ok ? 0u : 2u);
      tc_fence_before();
      named_bar_sync(1, 128);
      uint32_t v4[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) v4[w] = *reinterpret_cast<volatile uint32_t*>(&bars->vote[j & 1][w]);
      if ((v4[0] | v4[1] | v4[2] | v4[3]) & 2u) {
        failed = true;
        if (row == 0) record_failure(p, bars);
        break;
      }
      bool keep_h[2];
      if (p.half) {
        keep_h[0] = (j < nvis_h[0]) && !(skip_on && (v4[0] & v4[1] & 1u));
        keep_h[1] = (j < nvis_h[1]) && !(skip_on && (v4[2] & v4[3] & 1u));
      } else {
        keep_h[0] = keep_h[1] = !(skip_on && (v4[0] & v4[1] & v4[2] & v4[3] & 1u));
      }
      const bool tile_keep = keep_h[0] || keep_h[1];
      const bool my_keep = keep_h[half];
      if (leader && j < my_nvis) {
        if (!my_keep) {
          ++skipped;
          skip_word |= 1u << (j & 31);
        }
        if (p.skip_bits != nullptr && ((j & 31) == 31 || j == my_nvis - 1)) {
          const int qt = p.half ? 2 * pt + half : pt;
          p.skip_bits[((size_t)(b * p.Hq + hq) * p.nQ + qt) * p.nKw + (j >> 5)] = skip_word;
          skip_word = 0;
        }
      }
      if (row == 0) {
        bars->dec_word[j & 1] = tile_keep ? 1u : 0u;
        mbar_arrive(smem_u32(&bars->dec_ready[j & 1]));
        if (!tile_keep) mbar_arrive(smem_u32(&bars->p_ready[j & 1]));
      }
      if (!tile_keep) continue;

      uint32_t pk[BC / 2];
      if (my_keep) {
        const float m_new = fmaxf(m_true, m_tile);
        m_true = m_new;
        bool resc = false;
        if (m_ref == -INFINITY) m_ref = m_true;  // first kept key: O and l are still zero
        else resc = (m_true - m_ref) * p.scale_log2 > RESCALE_LOG2;
        if (__any_sync(0xffffffffu, resc)) {
          bool okw = (n_pv == 0) ||
                     mbar_wait(smem_u32(&bars->o_bar), (n_pv - 1) & 1, WAIT_TIMEOUT_NS);
          okw = __all_sync(0xffffffffu, okw);
          if (!okw) failed = true;  // reported at the next vote
          const float alpha = resc ? fast_exp2((m_ref - m_true) * p.scale_log2) : 1.f;
          if (okw && n_pv > 0) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(lane_base + O_COL + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(lane_base + O_COL + 32 * c, o);
            }
          }
          if (resc) {
            l *= alpha;
            m_ref = m_true;
          }
        }
        const float mref_s = (m_ref == -INFINITY) ? 0.f : m_ref * p.scale_log2;
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < BC; i += 2) {
          const float p0 = fast_exp2(fmaf(x[i], p.scale_log2, -mref_s));
          const float p1 = fast_exp2(fmaf(x[i + 1], p.scale_log2, -mref_s));
          lsum += p0 + p1;
          pk[i / 2] = pack_bf16x2(p0, p1);
        }
        l += lsum;
      } else {
#pragma unroll
        for (int i = 0; i < BC / 2; ++i) pk[i] = 0u;
      }
#pragma unroll
      for (int c = 0; c < BC / 64; ++c)
        tmem_st32(lane_base + S_COL + 128 * (j & 1) + 32 * c,
                  *reinterpret_cast<const uint32_t(*)[32]>(&pk[32 * c]));
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(2, 128);
      if (row == 0) mbar_arrive(smem_u32(&bars->p_ready[j & 1]));
      ++n_pv;
    }

    // ---- epilogue
    bool okf = true;
    if (nvis > 0) okf = mbar_wait(smem_u32(&bars->o_final), 0, WAIT_TIMEOUT_NS);
    okf = __all_sync(0xffffffffu, okf) && !failed;
    tc_fence_after();
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
    __nv_bfloat16* orow = p.out + ((size_t)(b * p.Lq + grow) * p.Hq + hq) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (okf && n_pv > 0) {
        tmem_ld32(lane_base + O_COL + 32 * c, o);
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
      p.lse[(size_t)(b * p.Hq + hq) * p.Lq + grow] =
          (l > 0.f) ? m_ref * p.scale + logf(l) : -INFINITY;
    if (leader) {
      const int qt = p.half ? 2 * pt + half : pt;
      if (qt < p.nQ) {
        p.skip_count[(size_t)(b * p.Hq + hq) * p.nQ + qt] = skipped;
        if (p.skip_bits != nullptr) {
          uint32_t* sb = p.skip_bits + ((size_t)(b * p.Hq + hq) * p.nQ + qt) * p.nKw;
          const int first_unwritten = (my_nvis + 31) / 32;
          for (int w = first_unwritten; w < p.nKw; ++w) sb[w] = 0u;
        }
      }
    }
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
static EncodeTiledFn g_encode = nullptr;
constexpr int MAX_DEV = 64;
static int* g_status[MAX_DEV] = {};
static bool g_attr_set[MAX_DEV][4] = {};

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

template <int D, int BC>
static int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const Params& p, int grid, cudaStream_t stream, int dev, int inst) {
  using L = Smem<D, BC>;
  if (!g_attr_set[dev][inst]) {
    if (cudaFuncSetAttribute(ssa_fwd_kernel<D, BC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::ALLOC) != cudaSuccess)
      return SSA_ERR_CUDA;
    g_attr_set[dev][inst] = true;
  }
  ssa_fwd_kernel<D, BC><<<grid, NTHREADS, L::ALLOC, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

static int run(const void* q, const void* k, const void* v, void* out, float* lse,
               int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
               float scale, int mode, float lambda, int n, int m, int sink, int recent, int Br,
               int Bc, void* stream, uint32_t* skip_bits, uint32_t* keep_bits) {
  // ---- argument checks (synchronous, nothing launched on failure)
  if (!q || !k || !v || !out || !lse || !tile_skip_count) return SSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Lk <= 0 || d <= 0) return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return SSA_ERR_INVALID_ARG;
  if (mode < 0 || mode > 3) return SSA_ERR_INVALID_ARG;
  if ((mode & SSA_MODE_SKIP) && (!std::isfinite(lambda) || lambda < 0.f)) return SSA_ERR_INVALID_ARG;
  if ((mode & SSA_MODE_NM) && (sink < 0 || recent < 0)) return SSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return SSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSA_ERR_UNSUPPORTED;
  if ((Br != 64 && Br != 128) || (Bc != 64 && Bc != 128)) return SSA_ERR_UNSUPPORTED;
  if (mode & SSA_MODE_NM) {
    if (!((m == 4 && n >= 1 && n <= 4) || (m == 8 && n >= 1 && n <= 8))) return SSA_ERR_UNSUPPORTED;
    if (Bc % m != 0) return SSA_ERR_UNSUPPORTED;
  }
  const long long nQp = (Lq + BM - 1) / BM;
  const long long grid = nQp * B * Hq;
  if (grid > 0x7fffffffLL) return SSA_ERR_UNSUPPORTED;
  if ((long long)B * Lq * Hq * d >= (1LL << 40) || (long long)B * Lk * Hkv * d >= (1LL << 40))
    return SSA_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEV) return SSA_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  Params p{};
  {
    std::lock_guard<std::mutex> g(g_mu);
    p.status = status_word(dev);
    if (!p.status) return SSA_ERR_CUDA;
    if (!make_map(&mq, q, B, Lq, Hq, d, BM) || !make_map(&mk, k, B, Lk, Hkv, d, Bc) ||
        !make_map(&mv, v, B, Lk, Hkv, d, Bc))
      return SSA_ERR_CUDA;
  }
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.skip_count = tile_skip_count;
  p.skip_bits = skip_bits;
  p.keep_bits = keep_bits;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk; p.causal = causal ? 1 : 0;
  p.mode = mode;
  p.n = (mode & SSA_MODE_NM) ? n : 0;
  p.m = (mode & SSA_MODE_NM) ? m : 4;
  p.sink = (mode & SSA_MODE_NM) ? sink : 0;
  p.recent = (mode & SSA_MODE_NM) ? recent : 0;
  p.half = (Br == 64) ? 1 : 0;
  p.Br = Br;
  p.nQp = (int)nQp;
  p.nQ = (Lq + Br - 1) / Br;
  p.nK = (Lk + Bc - 1) / Bc;
  p.nKw = (p.nK + 31) / 32;
  p.Lkw = (Lk + 31) / 32;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.log2_lambda = ((mode & SSA_MODE_SKIP) && lambda > 0.f) ? (float)std::log2((double)lambda)
                                                           : -INFINITY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> g(g_mu);
  if (d == 128 && Bc == 128) return launch<128, 128>(mq, mk, mv, p, (int)grid, st, dev, 0);
  if (d == 128 && Bc == 64) return launch<128, 64>(mq, mk, mv, p, (int)grid, st, dev, 1);
  if (d == 64 && Bc == 128) return launch<64, 128>(mq, mk, mv, p, (int)grid, st, dev, 2);
  return launch<64, 64>(mq, mk, mv, p, (int)grid, st, dev, 3);
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
                  uint32_t* keep_bits) {
  return ssa::run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, mode,
                  lambda, n, m, sink, recent, Br, Bc, stream, skip_bits, keep_bits);
}

int64_t ssa_visited_tiles(int causal, int Lq, int Lk, int Br, int Bc) {
  if (Lq <= 0 || Lk <= 0 || Br <= 0 || Bc <= 0) return -1;
  const int nQ = (Lq + Br - 1) / Br;
  int64_t t = 0;
  for (int qt = 0; qt < nQ; ++qt) t += ssa::visited_key_tiles(causal, Lq, Lk, Br, Bc, qt);
  return t;
}

int ssa_device_status(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SSA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= ssa::MAX_DEV) return SSA_ERR_CUDA;
  int* w;
  {
    std::lock_guard<std::mutex> g(ssa::g_mu);
    w = ssa::status_word(dev);
  }
  if (!w) return SSA_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SSA_ERR_CUDA;
  if (h != 0) {
    if (cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return SSA_ERR_CUDA;
    return SSA_ERR_TIMEOUT;
  }
  return SSA_OK;
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
