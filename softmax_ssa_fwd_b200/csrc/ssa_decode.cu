// ssa_decode.cu -- skip-softmax attention for decode (a few query rows per
// sequence against a long KV cache) on B200 (sm_100a), split over the keys.
//
// Method: "Skip-Softmax Sparse Attention for Diffusion Models" (intro,
// "Threshold Modes") and "Attention Sparsity for HuggingFace Models" (custom
// configuration: per-phase thresholds, prefill and decode; N:M applies to
// prefill only, so this path has no N:M).  A key tile is skipped for a query
// tile when exp(tile_row_max - running_max) < lambda for every row.
//
// Decode reads the whole KV cache for a handful of query rows, so it is bound
// by HBM; each sequence's key tiles are spread over `num_splits` CTAs per KV
// head.  Every split runs the skip-softmax recurrence over its own key tiles
// in order, with its own running max (its first tile is never skipped unless
// fully masked); a second kernel merges the splits' (max, sum, accumulator)
// with the usual log-sum-exp rule.  With one split this is exactly the
// prefill rule for a single query tile.
//
// Work item (split s, KV head, batch): the G = Hq / Hkv query heads that
// share the KV head, Lq rows each, R = G * Lq <= 32 rows in all, copied into
// each of the four 32-row lane quadrants of one 128-row query tile (the rest
// zero); a key tile is decided per query head (its Lq rows).  The kernel is
// persistent (one CTA per SM, each taking work items round-robin), so the
// loads of the next split stream in while the current one finishes.  256
// threads:
//   warp 0   producer: TMA loads of each key tile's K and V (128-byte swizzled
//            64-column boxes) into shared-memory rings (3 K tiles, 2 V
//            tiles: a K tile is free once its S is computed, a V tile only
//            after its P.V), ahead of the arithmetic and across splits.
//            Decode is bound by these bytes, so V is fetched with K: a
//            skipped tile saves its exponentials and P.V, not its V bytes.
//   warp 1   TMEM owner and MMA issuer: S = Q K^T into one of two S buffers
//            in TMEM, O += P V into one of two O buffers (one per split in
//            flight) with P read from TMEM, on tcgen05 (M = 128: the copies
//            cost tensor time, which decode has to spare, and no CUDA-core
//            arithmetic)
//   warps 2-3  query loader: the next split's query rows into the second of
//            two query tiles in shared memory
//   warps 4-7  softmax, one per lane quadrant, each on a quarter of the key
//            columns: masks, the tile row max (shared by the four warps),
//            the per-head vote (ballots), P -> TMEM as bf16 pairs, O rescale
//            when a row's max grows; each warp's quadrant of O and its row
//            sums are one partial result of the split, and the combine
//            kernel merges the four partials of every split with the splits
// Every wait is bounded; a wait that gives up raises the per-device status
// word that ssa_device_status reads.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/ssa.h"
#include "internal.h"
#include "ptx.cuh"

namespace ssa_dec {

using ssa::mbar_arrive;
using ssa::mbar_arrive_expect_tx;
using ssa::mbar_init;
using ssa::mbar_wait;
using ssa::smem_u32;

constexpr int NT = 256;          // warps 0 producer, 1 MMA, 2-3 query loader, 4-7 softmax
constexpr int RMAX = 32;         // query rows per split: one TMEM lane quadrant
constexpr int NPART = 4;         // partial results per split: one per softmax warp
constexpr int KST = 3;           // K ring depth (tiles)
constexpr int VST = 2;           // V ring depth (tiles)
constexpr uint32_t TMEM_COLS = 512;
// S of the CTA's g-th key tile (then its P) at columns [256 * (g & 1), + Bc):
// S_{g+1} is computed while the softmax of tile g runs
__device__ __forceinline__ uint32_t s_col(int g) { return 256u * (uint32_t)(g & 1); }
// O of the CTA's n-th split at columns [128 + 256 * (n & 1), + d): the next
// split accumulates while this one's O is read out
__device__ __forceinline__ uint32_t o_col(int n) { return 128u + 256u * (uint32_t)(n & 1); }
constexpr unsigned long long DRAIN_NS = 2000000000ull;

struct Params {
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  float* lse;
  int32_t* skip_count;
  float* o_part;    // [B, Hq, Lq, S * NPART, d]
  float* ml_part;   // [B, Hq, Lq, S * NPART, 2]: running max (log2 units), row sum
  int32_t* sk_part; // [B, Hq, S]
  uint32_t* skip_bits;  // optional [B, Hq, ceil(nK / 32)]: key tiles skipped (evidence output)
  int* status;
  unsigned long long wait_ns;
  int B, Hq, Hkv, Lq, Lk, causal, S, nK, tiles_per_split, G, R;
  int n_items;        // B * Hkv * S splits, handed out round-robin over the CTAs
  float c;            // scale * log2(e)
  float log2_lambda;  // -inf for lambda == 0
};

// The prefill TMA load with an L2 cache policy: the K/V stream is read once,
// and tagging it evict-first keeps the splits' partial results (written
// meanwhile, read by the combine kernel) in L2.
__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One split (work item): key tiles [kt0, kt0 + nt) of KV head hkv of sequence b.
struct Item {
  int s, hkv, b, kt0, nt;
};
__device__ __forceinline__ Item item_of(const Params& p, int it) {
  Item w;
  w.s = it % p.S;
  const int bh = it / p.S;
  w.hkv = bh % p.Hkv;
  w.b = bh / p.Hkv;
  w.kt0 = w.s * p.tiles_per_split;
  w.nt = max(0, min(p.nK, w.kt0 + p.tiles_per_split) - w.kt0);
  return w;
}

template <int D, int BC>
struct DecSmem {
  static constexpr uint32_t Q_BYTES = 128 * D * 2;         // one query tile, rows padded to 128
  static constexpr uint32_t TILE_BYTES = BC * D * 2;        // one K or V tile
  static constexpr uint32_t K_OFF = 2 * Q_BYTES;            // two query tiles: the next split's is loaded early
  static constexpr uint32_t V_OFF = K_OFF + KST * TILE_BYTES;
  static constexpr uint32_t TOTAL = 1024 + V_OFF + VST * TILE_BYTES;  // + alignment slack
};

// Persistent: CTA c takes splits c, c + gridDim.x, ... in turn.  Every role
// walks the same sequence of splits; the K/V ring, the S buffers and their
// barriers run on per-CTA tile counters across splits, so the loads of the
// next split overlap the end of the current one.
template <int D, int BC>
__global__ void __launch_bounds__(NT, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const Params p) {
  using L = DecSmem<D, BC>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* q_tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t kfull[KST], kempty[KST], vfull[VST], vempty[VST];
  __shared__ uint64_t q_full[2], q_empty[2], s_full[2], p_ready[2], pv_done, o_done[2], mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ uint32_t keep_word[2];            // tile decision for the MMA warp, by tile parity
  __shared__ float red_max[2][4][32];          // per-warp row maxima, by tile parity

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G, R = p.R, Lq = p.Lq;

  if (tid == 0) {
    for (int i = 0; i < KST; ++i) {
      mbar_init(smem_u32(&kfull[i]), 1);
      mbar_init(smem_u32(&kempty[i]), 1);
    }
    for (int i = 0; i < VST; ++i) {
      mbar_init(smem_u32(&vfull[i]), 1);
      mbar_init(smem_u32(&vempty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&q_full[i]), 64);  // every thread of the two loader warps
      mbar_init(smem_u32(&q_empty[i]), 1);
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&o_done[i]), 1);
      // P of the CTA's tiles 2m + i: one arrival per softmax warp.  One
      // barrier per tile parity, like S: the softmax can finish tile g + 1
      // (and, once S_{g+2} is issued, g + 2) before the MMA warp has looked
      // at tile g + 1's phase
      mbar_init(smem_u32(&p_ready[i]), 4);
    }
    mbar_init(smem_u32(&pv_done), 1);
    mbar_init(smem_u32(&mma_done), 1);
    ssa::fence_mbar_init();
  }
  if (warp == 1) {
    ssa::tmem_alloc(smem_u32(&tmem_base), TMEM_COLS);
    ssa::tmem_relinquish();
  }
  // both query tiles zero: rows R..127 stay zero for every split
  for (int e = tid; e < (int)(2 * L::Q_BYTES / 16); e += NT)
    reinterpret_cast<uint4*>(q_tiles)[e] = make_uint4(0u, 0u, 0u, 0u);
  ssa::fence_proxy_async_smem();  // generic writes of the tiles, then tensor-core reads
  ssa::tc_fence_before();
  __syncthreads();
  ssa::tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t q_s = smem_u32(q_tiles), k_ring = q_s + L::K_OFF, v_ring = q_s + L::V_OFF;

  if (warp == 0) {
    // ======================= producer: K and V tiles by TMA =======================
    if (lane == 0) {
      ssa::tma_prefetch_desc(&tm_k);
      ssa::tma_prefetch_desc(&tm_v);
      const uint64_t stream_policy = l2_evict_first_policy();
      int g = 0, kdone = 0, vdone = 0;  // tiles walked; K and V tiles issued
      bool ok = true;
      for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
        const Item w = item_of(p, it);
        for (int t = 0; t < w.nt; ++t, ++g) {
          const int j0 = (w.kt0 + t) * BC;
          const int ks = g % KST, vs = g % VST;
          if (!mbar_wait(smem_u32(&kempty[ks]), ((g / KST) & 1) ^ 1, p.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t kb = smem_u32(&kfull[ks]);
          mbar_arrive_expect_tx(kb, L::TILE_BYTES);
#pragma unroll
          for (int box = 0; box < D / 64; ++box)
            tma_load_4d_hint(k_ring + ks * L::TILE_BYTES + box * BC * 128, &tm_k, kb, box * 64, w.hkv, j0, w.b,
                             stream_policy);
          kdone = g + 1;
          if (!mbar_wait(smem_u32(&vempty[vs]), ((g / VST) & 1) ^ 1, p.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t vb = smem_u32(&vfull[vs]);
          mbar_arrive_expect_tx(vb, L::TILE_BYTES);
#pragma unroll
          for (int box = 0; box < D / 64; ++box)
            tma_load_4d_hint(v_ring + vs * L::TILE_BYTES + box * BC * 128, &tm_v, vb, box * 64, w.hkv, j0, w.b,
                             stream_policy);
          vdone = g + 1;
        }
      }
      if (!ok) atomicOr(p.status, 1);
      // drain: every load issued has landed before the CTA may exit
      bool drained = true;
      for (int t = max(0, kdone - KST); t < kdone; ++t)
        drained &= mbar_wait(smem_u32(&kfull[t % KST]), (t / KST) & 1, DRAIN_NS);
      for (int t = max(0, vdone - VST); t < vdone; ++t)
        drained &= mbar_wait(smem_u32(&vfull[t % VST]), (t / VST) & 1, DRAIN_NS);
      if (!drained) atomicOr(p.status, 1);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = ssa::idesc_bf16_f32(128, BC, false, false);
      constexpr uint32_t idesc_pv = ssa::idesc_bf16_f32(128, D, false, true);
      // cursor of the S stream: split it_s (its n_s-th non-empty one), its tile t_s; g_s tiles so far
      int it_s = blockIdx.x, t_s = 0, n_s = 0, g_s = 0;
      Item w_s{};
      auto seek = [&](int& it, Item& w) {
        for (; it < p.n_items; it += gridDim.x) {
          w = item_of(p, it);
          if (w.nt > 0) break;
        }
      };
      seek(it_s, w_s);
      // S_g = Q K_g^T into TMEM columns [s_col(g), s_col(g) + BC)
      auto issue_s = [&]() -> bool {
        const int qb = n_s & 1;
        if (t_s == 0 && !mbar_wait(smem_u32(&q_full[qb]), (n_s >> 1) & 1, p.wait_ns)) return false;
        const int ks = g_s % KST;
        if (!mbar_wait(smem_u32(&kfull[ks]), (g_s / KST) & 1, p.wait_ns)) return false;
        ssa::tc_fence_after();
        const uint32_t k_s = k_ring + ks * L::TILE_BYTES, qt = q_s + qb * L::Q_BYTES;
#pragma unroll
        for (int k16 = 0; k16 < D / 16; ++k16) {
          const uint32_t qoff = (k16 >> 2) * (128 * 128) + (k16 & 3) * 32;
          const uint32_t koff = (k16 >> 2) * (BC * 128) + (k16 & 3) * 32;
          ssa::mma_ss(tmem + s_col(g_s), ssa::smem_desc_sw128(qt + qoff, 16, 1024),
                      ssa::smem_desc_sw128(k_s + koff, 16, 1024), idesc_qk, k16 > 0 ? 1u : 0u);
        }
        ssa::mma_commit(smem_u32(&s_full[g_s & 1]));
        ssa::mma_commit(smem_u32(&kempty[ks]));  // the K tile is free once S_g is done
        if (++t_s == w_s.nt) {
          ssa::mma_commit(smem_u32(&q_empty[qb]));  // and the query tile after the split's last S
          t_s = 0;
          ++n_s;
          it_s += gridDim.x;
          seek(it_s, w_s);
        }
        ++g_s;
        return true;
      };
      bool ok = true;
      for (int i = 0; ok && i < 2 && it_s < p.n_items; ++i) ok = issue_s();
      // cursor of the P.V stream
      int it_p = blockIdx.x, t_p = 0, n_p = 0, g_p = 0, pv_count = 0;
      Item w_p{};
      seek(it_p, w_p);
      while (ok && it_p < p.n_items) {
        const int vs = g_p % VST;
        if (!mbar_wait(smem_u32(&p_ready[g_p & 1]), (g_p >> 1) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        // the V tile has to have landed before its slot is handed back, kept or not
        if (!mbar_wait(smem_u32(&vfull[vs]), (g_p / VST) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        if (*reinterpret_cast<volatile uint32_t*>(&keep_word[g_p & 1])) {
          // O += P V: P (bf16 pairs over the S columns) from TMEM, V from the stage
          ssa::tc_fence_after();
          const uint32_t v_s = v_ring + vs * L::TILE_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < BC / 16; ++k16)
            ssa::mma_ts(tmem + o_col(n_p), tmem + s_col(g_p) + k16 * 8,
                        ssa::smem_desc_sw128(v_s + k16 * 16 * 128, BC * 128, 1024), idesc_pv,
                        (pv_count > 0 || k16 > 0) ? 1u : 0u);
          ++pv_count;
        }
        ssa::mma_commit(smem_u32(&vempty[vs]));  // the V tile is free once these MMAs are done
        ssa::mma_commit(smem_u32(&pv_done));     // O holds every P.V up to this tile
        if (++t_p == w_p.nt) {
          // the split's O is complete (the softmax read the previous O in
          // this buffer before it handed over any P of this split)
          ssa::mma_commit(smem_u32(&o_done[n_p & 1]));
          t_p = 0;
          pv_count = 0;
          ++n_p;
          it_p += gridDim.x;
          seek(it_p, w_p);
        }
        ++g_p;
        // (S_{g+2} overwrites P_g: it follows the P.V in issue order)
        if (it_s < p.n_items) ok = issue_s();
      }
      if (!ok) atomicOr(p.status, 1);
      ssa::mma_commit(smem_u32(&mma_done));
      if (!mbar_wait(smem_u32(&mma_done), 0, DRAIN_NS)) atomicOr(p.status, 1);
    }
  } else if (warp == 2 || warp == 3) {
    // ======================= query loader: the next split's rows =======================
    // row r = g * Lq + i (head hkv * G + g, query row i), copied to rows r,
    // 32 + r, 64 + r and 96 + r (one copy per TMEM lane quadrant, so each
    // softmax warp sees every row); K-major with 128-byte swizzle, as the
    // MMA's A operand
    const int lt = tid - 64;
    int n = 0;
    for (int it = blockIdx.x; it < p.n_items; it += gridDim.x) {
      const Item w = item_of(p, it);
      if (w.nt == 0) continue;
      const int qb = n & 1;
      if (!mbar_wait(smem_u32(&q_empty[qb]), ((n >> 1) & 1) ^ 1, p.wait_ns)) {
        if (lt == 0) atomicOr(p.status, 1);
        break;
      }
      uint8_t* qt = q_tiles + qb * L::Q_BYTES;
      for (int e = lt; e < R * (D / 8); e += 64) {
        const int r = e / (D / 8), u = e % (D / 8);
        const int g = r / Lq, i = r % Lq;
        const uint4 val =
            *reinterpret_cast<const uint4*>(p.q + (((size_t)w.b * Lq + i) * p.Hq + w.hkv * G + g) * D + 8 * u);
        const int box = u >> 3, unit = u & 7;
#pragma unroll
        for (int cp = 0; cp < 4; ++cp)  // rows 32 cp + r: same swizzle phase (r & 7)
          *reinterpret_cast<uint4*>(qt + box * 128 * 128 + (32 * cp + r) * 128 + ((unit ^ (r & 7)) << 4)) = val;
      }
      ssa::fence_proxy_async_smem();
      mbar_arrive(smem_u32(&q_full[qb]));
      ++n;
    }
  } else if (warp >= 4) {
    // ======================= softmax =======================
    // Warp 4 + qd owns TMEM lanes [32 qd, 32 qd + 32) (its copy of the query
    // rows: lane r = row r) and key columns [qd * CW, qd * CW + CW) of every
    // tile.  The four warps share each row's tile max (so every warp takes
    // the same skip decisions and uses the same running max), and each keeps
    // its own row sums and, in its lane quadrant of O, its own accumulator:
    // the four partial results of a split are merged with the splits.
    constexpr int CW = BC / 4;
    const int qd = warp - 4;
    const uint32_t tq = tmem + ((uint32_t)(32 * qd) << 16);
    const int r = lane;
    const bool valid = r < R;
    const int g = valid ? r / Lq : 0, i = valid ? r % Lq : 0;
    const int pos = i + p.Lk - Lq;
    const uint32_t head_mask = ((Lq >= 32) ? 0xffffffffu : ((1u << Lq) - 1u)) << ((lane < G ? lane : 0) * Lq);
    uint32_t zero[CW / 2];
#pragma unroll
    for (int e = 0; e < CW / 2; ++e) zero[e] = 0u;
    int gt = 0, n = 0;  // tiles and non-empty splits so far
    bool failed = false;
    for (int it = blockIdx.x; it < p.n_items; it += gridDim.x) {
      const Item w = item_of(p, it);
      const uint32_t oc = o_col(n);
      float m_true = -INFINITY, l = 0.f;  // log2 units of scale * q.k
      int n_pv = 0, skipped = 0;
      for (int t = 0; t < w.nt; ++t, ++gt) {
        bool ok = !failed && mbar_wait(smem_u32(&s_full[gt & 1]), (gt >> 1) & 1, p.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && !failed) {
          if (lane == 0) atomicOr(p.status, 1);
          failed = true;
        }
        ssa::tc_fence_after();
        float x[CW];
        if constexpr (CW == 32) ssa::tmem_ld32f(tq + s_col(gt) + qd * CW, x);
        else ssa::tmem_ld16f(tq + s_col(gt) + qd * CW, x);
        ssa::tmem_wait_ld();
        const int j0 = (w.kt0 + t) * BC + qd * CW;  // first key of this warp's columns
        int lim = p.Lk - 1 - j0;  // last visible key of this row, relative to j0
        if (p.causal && pos - j0 < lim) lim = pos - j0;
        if (!valid || !ok) lim = -1;
        float ml = -INFINITY;
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          x[c] = (c > lim) ? -INFINITY : x[c] * p.c;
          ml = fmaxf(ml, x[c]);
        }
        // the row's max over the whole tile: the four warps' maxima
        volatile float* rm = &red_max[gt & 1][0][0];
        rm[32 * qd + lane] = ml;
        ssa::named_bar_sync(1, 128);
        const float mt = fmaxf(fmaxf(rm[lane], rm[32 + lane]), fmaxf(rm[64 + lane], rm[96 + lane]));
        const bool neg = mt == -INFINITY || (m_true != -INFINITY && (mt - m_true) < p.log2_lambda);
        const uint32_t negs = __ballot_sync(0xffffffffu, neg || !valid);
        // lane g < G holds head g's decision; every row reads its own head's
        const bool head_keeps = lane < G && (negs & head_mask) != head_mask;
        const uint32_t keeps = __ballot_sync(0xffffffffu, head_keeps);
        if (lane < G && !head_keeps) {
          ++skipped;
          if (p.skip_bits != nullptr && qd == 0) {
            const int kt = w.kt0 + t;
            atomicOr(p.skip_bits + ((size_t)w.b * p.Hq + w.hkv * G + lane) * ((p.nK + 31) / 32) + (kt >> 5),
                     1u << (kt & 31));
          }
        }
        const bool mine = valid && ((keeps >> g) & 1u);
        if (keeps != 0u) {
          const float m_new = fmaxf(m_true, mt);
          const bool grow = mine && m_true != -INFINITY && m_new > m_true;
          const float alpha = grow ? ex2(m_true - m_new) : 1.f;
          const float mref = (m_new == -INFINITY) ? 0.f : m_new;
          float sum = 0.f;
          uint32_t pk[CW / 2];
#pragma unroll
          for (int c2 = 0; c2 < CW / 2; ++c2) {
            const float p0 = mine ? ex2(x[2 * c2] - mref) : 0.f;
            const float p1 = mine ? ex2(x[2 * c2 + 1] - mref) : 0.f;
            sum += p0 + p1;
            __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            pk[c2] = *reinterpret_cast<uint32_t*>(&pb);
          }
          // P over the tile's columns (bf16 pairs): this warp's keys, zero for
          // the other warps' keys
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {
            const uint32_t col = tq + s_col(gt) + blk * (CW / 2);
            if constexpr (CW == 32) ssa::tmem_st16(col, blk == qd ? pk : zero);
            else ssa::tmem_st8(col, blk == qd ? pk : zero);
          }
          if (__any_sync(0xffffffffu, grow) && n_pv > 0) {
            // rescale this quadrant of O once every earlier P.V has finished
            // (S_g was issued after the P.V of tile g - 2, so at most tile
            // g - 1's is out)
            bool done = !failed && mbar_wait(smem_u32(&pv_done), (gt - 1) & 1, p.wait_ns);
            done = __all_sync(0xffffffffu, done);
            if (!done && !failed) {
              if (lane == 0) atomicOr(p.status, 1);
              failed = true;
            }
            ssa::tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              ssa::tmem_ld32(tq + oc + 32 * cc, o);
              ssa::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              ssa::tmem_st32(tq + oc + 32 * cc, o);
            }
          }
          if (mine) {
            l = l * alpha + sum;
            m_true = m_new;
          }
          ++n_pv;
        }
        ssa::tmem_wait_st();
        if (qd == 0 && lane == 0) *reinterpret_cast<volatile uint32_t*>(&keep_word[gt & 1]) = keeps != 0u ? 1u : 0u;
        ssa::tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_ready[gt & 1]));
      }
      // ---- end of the split: this warp's unnormalised accumulator and (max, sum) per row
      bool okf = true;
      if (w.nt > 0) {
        okf = !failed && mbar_wait(smem_u32(&o_done[n & 1]), (n >> 1) & 1, p.wait_ns);
        ++n;
      }
      okf = __all_sync(0xffffffffu, okf) && !failed;
      if (!okf && !failed) {
        if (lane == 0) atomicOr(p.status, 1);
        failed = true;
      }
      ssa::tc_fence_after();
      const int hq = w.hkv * G + g;
      const size_t part = (((size_t)w.b * p.Hq + hq) * Lq + i) * ((size_t)p.S * NPART) + (size_t)w.s * NPART + qd;
      float* orow = p.o_part + part * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (okf && n_pv > 0) {
          ssa::tmem_ld32(tq + oc + 32 * cc, o);
          ssa::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4)
            reinterpret_cast<float4*>(orow + 32 * cc)[e4] =
                make_float4(__uint_as_float(o[4 * e4]), __uint_as_float(o[4 * e4 + 1]),
                            __uint_as_float(o[4 * e4 + 2]), __uint_as_float(o[4 * e4 + 3]));
        }
      }
      if (valid) {
        float* mlp = p.ml_part + part * 2;
        mlp[0] = m_true;
        mlp[1] = (okf && n_pv > 0) ? l : 0.f;
      }
      if (qd == 0 && lane < G) p.sk_part[((size_t)w.b * p.Hq + w.hkv * G + lane) * p.S + w.s] = skipped;
    }
  }

  // ---- teardown
  ssa::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ssa::tc_fence_after();
    ssa::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Merge the partial results of one (batch, head, query row): S * NPART of
// them, by the log-sum-exp rule.  2 * d threads: first the largest max among
// the partials that kept a key (all threads), then four groups of d / 2
// threads (two columns each) sum every fourth partial, and group 0 adds the
// four group sums.
template <int D>
__global__ void __launch_bounds__(2 * D) decode_combine_kernel(const Params p) {
  constexpr int TPG = D / 2, NG = 4, NW = 2 * D / 32;
  __shared__ float wmax[NW];
  __shared__ float gacc[NG][D];
  __shared__ float gsum[NG];
  const int i = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, grp = tid / TPG, t = tid % TPG;
  const size_t row = ((size_t)b * p.Hq + hq) * p.Lq + i;
  const int np = p.S * NPART;
  const float* ml = p.ml_part + row * np * 2;
  float mx = -INFINITY;
  for (int s = tid; s < np; s += 2 * D)
    if (ml[2 * s + 1] > 0.f) mx = fmaxf(mx, ml[2 * s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = mx;
  __syncthreads();
  float M = wmax[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, wmax[w]);
  // a partial that kept no key has l = 0 and an all-zero accumulator
  float L = 0.f, a0 = 0.f, a1 = 0.f;
  const float* ob = p.o_part + row * (size_t)np * D + 2 * t;
#pragma unroll 4
  for (int s = grp; s < np; s += NG) {
    const float ls = ml[2 * s + 1];
    const float w = ls > 0.f ? ex2(ml[2 * s] - M) : 0.f;
    const float2 o = *reinterpret_cast<const float2*>(ob + (size_t)s * D);
    L = fmaf(w, ls, L);
    a0 = fmaf(w, o.x, a0);
    a1 = fmaf(w, o.y, a1);
  }
  gacc[grp][2 * t] = a0;
  gacc[grp][2 * t + 1] = a1;
  if (t == 0) gsum[grp] = L;
  __syncthreads();
  if (grp != 0) return;
  a0 = gacc[0][2 * t] + gacc[1][2 * t] + gacc[2][2 * t] + gacc[3][2 * t];
  a1 = gacc[0][2 * t + 1] + gacc[1][2 * t + 1] + gacc[2][2 * t + 1] + gacc[3][2 * t + 1];
  L = gsum[0] + gsum[1] + gsum[2] + gsum[3];
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat162 res = __floats2bfloat162_rn(a0 * inv, a1 * inv);
  *reinterpret_cast<__nv_bfloat162*>(p.out + (((size_t)b * p.Lq + i) * p.Hq + hq) * D + 2 * t) = res;
  if (t == 0) {
    p.lse[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    if (i == 0) {
      int sum = 0;
      for (int s = 0; s < p.S; ++s) sum += p.sk_part[((size_t)b * p.Hq + hq) * p.S + s];
      p.skip_count[(size_t)b * p.Hq + hq] = sum;
    }
  }
}

template <int D, int BC>
static int launch_bc(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, cudaStream_t st) {
  using L = DecSmem<D, BC>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SSA_ERR_CUDA;
  int n_sm = 0;
  {
    // per instance and device, once before the first launch there; callers may be threads
    static std::mutex mu;
    static bool attr_set[64] = {};
    static int sms[64] = {};
    std::lock_guard<std::mutex> g(mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(decode_split_kernel<D, BC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)L::TOTAL) != cudaSuccess)
        return SSA_ERR_CUDA;
      attr_set[dev] = true;
    }
    if (!sms[dev]) {
      int v = 0;
      if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        return SSA_ERR_CUDA;
      sms[dev] = v;
    }
    n_sm = sms[dev];
  }
  const int grid = p.n_items < n_sm ? p.n_items : n_sm;  // one CTA per SM, persistent
  decode_split_kernel<D, BC><<<grid, NT, L::TOTAL, st>>>(mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return SSA_ERR_CUDA;
  decode_combine_kernel<D><<<dim3(p.Lq, p.Hq, p.B), 2 * D, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

static size_t workspace_bytes(int B, int Hq, int Lq, int d, int S) {
  const size_t rows = (size_t)B * Hq * Lq, parts = (size_t)S * NPART;
  return rows * parts * d * sizeof(float) + rows * parts * 2 * sizeof(float) + (size_t)B * Hq * S * sizeof(int32_t);
}

}  // namespace ssa_dec

extern "C" {

size_t ssa_decode_workspace_bytes(int B, int Hq, int Lq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || Lq <= 0 || d <= 0 || num_splits <= 0) return 0;
  return ssa_dec::workspace_bytes(B, Hq, Lq, d, num_splits);
}

int ssa_decode_default_splits(int B, int Hkv, int Lk, int Bc, int num_sms) {
  if (B <= 0 || Hkv <= 0 || Lk <= 0 || (Bc != 64 && Bc != 128) || num_sms <= 0) return 0;
  const long long pairs = (long long)B * Hkv;
  const int nK = (int)(((long long)Lk + Bc - 1) / Bc);
  const int smax = nK < 256 ? nK : 256;
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= smax; ++s) {
    const int T = (nK + s - 1) / s;  // key tiles per split
    if ((nK + T - 1) / T < s) continue;  // would leave empty splits: a smaller count does the same
    const long long rounds = (pairs * s + num_sms - 1) / num_sms;  // items of the busiest CTA
    const long long cost = rounds * (T + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

static int decode_run(const void* q, const void* k, const void* v, void* out, float* lse,
                      int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
                      float scale, float lambda, int Bc, int num_splits, void* workspace,
                      size_t workspace_bytes, void* stream, uint32_t* skip_bits) {
  using namespace ssa_dec;
  if (!q || !k || !v || !out || !lse || !tile_skip_count || !workspace) return SSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(tile_skip_count) | reinterpret_cast<uintptr_t>(skip_bits) |
       reinterpret_cast<uintptr_t>(lse)) & 3u)
    return SSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Lk <= 0 || d <= 0 || num_splits <= 0)
    return SSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SSA_ERR_INVALID_ARG;
  if (!(lambda >= 0.f) || !std::isfinite(lambda)) return SSA_ERR_INVALID_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out) |
                        reinterpret_cast<uintptr_t>(workspace);
  if (mis & 15u) return SSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSA_ERR_UNSUPPORTED;
  if (Bc != 64 && Bc != 128) return SSA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G * Lq > RMAX) return SSA_ERR_UNSUPPORTED;
  if (workspace_bytes < ssa_dec::workspace_bytes(B, Hq, Lq, d, num_splits)) return SSA_ERR_INVALID_ARG;

  Params p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.skip_count = tile_skip_count;
  p.skip_bits = skip_bits;
  const size_t rows = (size_t)B * Hq * Lq;
  p.o_part = static_cast<float*>(workspace);
  p.ml_part = p.o_part + rows * num_splits * NPART * d;
  p.sk_part = reinterpret_cast<int32_t*>(p.ml_part + rows * num_splits * NPART * 2);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lk = Lk;
  p.causal = causal ? 1 : 0;
  p.S = num_splits;
  p.nK = (Lk + Bc - 1) / Bc;
  p.tiles_per_split = (p.nK + num_splits - 1) / num_splits;
  if ((long long)B * Hkv * num_splits > (1LL << 30)) return SSA_ERR_UNSUPPORTED;
  p.n_items = B * Hkv * num_splits;
  p.G = G;
  p.R = G * Lq;
  p.c = (float)((double)scale * 1.4426950408889634);
  p.log2_lambda = lambda > 0.f ? log2f(lambda) : -INFINITY;
  if ((long long)B * Lk * Hkv * d >= (1LL << 40)) return SSA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SSA_ERR_CUDA;
  p.status = ssa::device_status_word(dev);
  if (!p.status) return SSA_ERR_CUDA;
  p.wait_ns = ssa::wait_timeout_ns();
  CUtensorMap mk, mv;
  if (!ssa::tma_map_bf16(&mk, k, B, Lk, Hkv, d, Bc) || !ssa::tma_map_bf16(&mv, v, B, Lk, Hkv, d, Bc))
    return SSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128) return Bc == 128 ? launch_bc<128, 128>(mk, mv, p, st) : launch_bc<128, 64>(mk, mv, p, st);
  return Bc == 128 ? launch_bc<64, 128>(mk, mv, p, st) : launch_bc<64, 64>(mk, mv, p, st);
}

int ssa_decode(const void* q, const void* k, const void* v, void* out, float* lse,
               int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
               float scale, float lambda, int Bc, int num_splits, void* workspace,
               size_t workspace_bytes, void* stream) {
  return decode_run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, lambda,
                    Bc, num_splits, workspace, workspace_bytes, stream, nullptr);
}

int ssa_decode_debug(const void* q, const void* k, const void* v, void* out, float* lse,
                     int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
                     float scale, float lambda, int Bc, int num_splits, void* workspace,
                     size_t workspace_bytes, void* stream, uint32_t* skip_bits) {
  if (!skip_bits) return SSA_ERR_INVALID_ARG;
  return decode_run(q, k, v, out, lse, tile_skip_count, B, Hq, Hkv, Lq, Lk, d, causal, scale, lambda,
                    Bc, num_splits, workspace, workspace_bytes, stream, skip_bits);
}

}  // extern "C"
