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
// by HBM; the arithmetic runs on the CUDA cores and each sequence's key tiles
// are spread over `num_splits` CTAs per KV head.  Every split runs the
// skip-softmax recurrence over its own key tiles in order, with its own
// running max (its first tile is never skipped unless fully masked); a second
// kernel merges the splits' (max, sum, accumulator) with the usual
// log-sum-exp rule.  With one split this is exactly the prefill rule for a
// single query tile.
//
// CTA (split s, KV head, batch): the G = Hq / Hkv query heads that share the
// KV head, Lq rows each, R = G * Lq <= 32 rows in all; a key tile is decided
// per query head (its Lq rows).  288 threads:
//   warp 8     producer: TMA loads of each key tile's K and V (128-byte
//              swizzled 64-column boxes) into an NS-stage shared-memory ring,
//              running up to NS tiles ahead of the arithmetic.  Decode is
//              bound by these bytes, so V is fetched with K: a skipped tile
//              saves its exponentials and P.V, not its V bytes.
//   warps 0-7  scores: thread t takes key t / TPK and a 1/TPK slice of d from
//              shared memory, q.k against all R rows (packed fp32x2 FMAs),
//              slices combined by shuffles; softmax: warp w owns rows w,
//              w + 8, ...: tile row max, vote, P, row sum; P.V: each thread
//              two output columns and every (256 / (d/2))-th key of the tile,
//              partial accumulators of all R rows in registers, summed over
//              threads through shared memory at the end of the split.
// Every wait is bounded; a wait that gives up raises the per-device status
// word that ssa_device_status reads.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/ssa.h"
#include "internal.h"
#include "ptx.cuh"

namespace ssa_dec {

using ssa::mbar_arrive;
using ssa::mbar_arrive_expect_tx;
using ssa::mbar_init;
using ssa::mbar_wait;
using ssa::smem_u32;

constexpr int NTC = 256;         // arithmetic threads (warps 0-7)
constexpr int NT = NTC + 32;     // plus the producer warp
constexpr int RMAX = 32;
constexpr int NS = 3;            // K/V ring depth (tiles)
constexpr uint32_t COMPUTE_BAR = 1;  // named barrier of the 256 arithmetic threads
constexpr unsigned long long DRAIN_NS = 2000000000ull;

struct Params {
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  float* lse;
  int32_t* skip_count;
  float* o_part;    // [B, Hq, Lq, S, d]
  float* ml_part;   // [B, Hq, Lq, S, 2]: running max (log2 units), row sum
  int32_t* sk_part; // [B, Hq, S]
  int* status;
  unsigned long long wait_ns;
  int B, Hq, Hkv, Lq, Lk, causal, S, nK, tiles_per_split, G, R;
  float c;            // scale * log2(e)
  float log2_lambda;  // -inf for lambda == 0
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync %0, %1;" ::"r"(COMPUTE_BAR), "r"(NTC) : "memory");
}

template <int D, int BC>
struct DecSmem {
  static constexpr uint32_t TILE_BYTES = BC * D * 2;        // one K or V tile
  static constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;   // K then V
  static constexpr uint32_t RING_BYTES = NS * STAGE_BYTES;
};

// Byte offset of element (row, col) of a [D/64 boxes][rows][64] tile written by
// TMA with 128-byte swizzle: 16-byte unit u of row r lands at u ^ (r & 7).
template <int BC>
__device__ __forceinline__ uint32_t sw128(int row, int col) {
  const int box = col >> 6, inrow = (col & 63) * 2;
  return (uint32_t)(box * BC * 128 + row * 128 + ((((inrow >> 4) ^ row) & 7) << 4) + (inrow & 15));
}

template <int D, int BC, int RT>
__global__ void __launch_bounds__(NT, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const Params p) {
  constexpr int TPK = NTC / BC;      // threads per key in the score phase
  constexpr int DP = D / TPK;        // d slice per thread
  constexpr int QP = DP + 4;         // padded slice stride: slices of a row start in different banks
  constexpr int QSTR = TPK * QP;     // q row stride in shared memory
  constexpr int NDP = D / 2;         // column pairs
  constexpr int NKG = NTC / NDP;     // key groups in the P.V phase
  using L = DecSmem<D, BC>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  float* qs = reinterpret_cast<float*>(ring + L::RING_BYTES);  // RT * QSTR; reused for the O reduction
  float* ss = qs + RT * QSTR;                                   // RT * BC scores, then P
  __shared__ float alpha_s[RT];
  __shared__ float mt_s[RT];
  __shared__ int neg_s[RT];
  __shared__ int keep_s[RMAX];  // per query head
  __shared__ int any_keep_s;
  __shared__ uint64_t full_bar[NS], empty_bar[NS];
  __shared__ int failed_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int G = p.G, R = p.R, Lq = p.Lq;
  const int kt0 = s * p.tiles_per_split;
  const int kt1 = min(p.nK, kt0 + p.tiles_per_split);
  const int ntiles = max(0, kt1 - kt0);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 8);  // one arrival per arithmetic warp
    }
    failed_s = 0;
    ssa::fence_mbar_init();
  }
  __syncthreads();

  if (warp == 8) {
    // ======================= producer =======================
    if (lane == 0 && ntiles > 0) {
      ssa::tma_prefetch_desc(&tm_k);
      ssa::tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % NS;
        if (!mbar_wait(smem_u32(&empty_bar[st]), ((t / NS) & 1) ^ 1, p.wait_ns)) {
          atomicOr(p.status, 1);
          *reinterpret_cast<volatile int*>(&failed_s) = 1;
          break;
        }
        const uint32_t fb = smem_u32(&full_bar[st]);
        mbar_arrive_expect_tx(fb, L::STAGE_BYTES);
        const uint32_t kd = smem_u32(ring + st * L::STAGE_BYTES), vd = kd + L::TILE_BYTES;
        const int j0 = (kt0 + t) * BC;
#pragma unroll
        for (int box = 0; box < D / 64; ++box) {
          ssa::tma_load_4d(kd + box * BC * 128, &tm_k, fb, box * 64, hkv, j0, b);
          ssa::tma_load_4d(vd + box * BC * 128, &tm_v, fb, box * 64, hkv, j0, b);
        }
        issued = t + 1;
      }
      // drain: every load issued has landed before the CTA may exit
      bool drained = true;
      for (int t = max(0, issued - NS); t < issued; ++t)
        drained &= mbar_wait(smem_u32(&full_bar[t % NS]), (t / NS) & 1, DRAIN_NS);
      if (!drained) atomicOr(p.status, 1);
    }
    return;
  }

  // ======================= arithmetic warps =======================
  // q rows: r = g * Lq + i -> head hkv * G + g, query row i
  for (int e = tid; e < RT * D; e += NTC) {
    const int r = e / D, dd = e % D;
    float val = 0.f;
    if (r < R) {
      const int g = r / Lq, i = r % Lq;
      val = __bfloat162float(p.q[(((size_t)b * Lq + i) * p.Hq + hkv * G + g) * D + dd]) * p.c;
    }
    qs[r * QSTR + (dd / DP) * QP + dd % DP] = val;
  }
  // per-row state, owned by warp r % 8 (every lane holds a copy)
  float m_run[RT / 8 > 0 ? RT / 8 : 1], l_run[RT / 8 > 0 ? RT / 8 : 1];
#pragma unroll
  for (int u = 0; u < (RT / 8 > 0 ? RT / 8 : 1); ++u) {
    m_run[u] = -INFINITY;
    l_run[u] = 0.f;
  }
  const int dpair = tid % NDP, kg = tid / NDP;
  float o0[RT], o1[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) o0[r] = o1[r] = 0.f;
  int skipped_tiles = 0;  // per head, kept by thread g (< G)
  bool failed = false;
  compute_sync();

  const int kc = tid / TPK, kpart = tid % TPK;
  for (int t = 0; t < ntiles; ++t) {
    const int kt = kt0 + t;
    const int j0 = kt * BC;
    const int st = t % NS;
    bool ok = !failed && mbar_wait(smem_u32(&full_bar[st]), (t / NS) & 1, p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && !failed) {
      if (lane == 0) atomicOr(p.status, 1);
      failed = true;
    }
    const uint8_t* ks = ring + st * L::STAGE_BYTES;
    const uint8_t* vs = ks + L::TILE_BYTES;
    // ---- scores: ss[r][c] = q_r . k_{j0+c} in log2 units (-inf where masked)
    {
      const int c = kc, part = kpart;
      const int j = j0 + c;
      float kv[DP];
#pragma unroll
      for (int u = 0; u < DP / 8; ++u) {
        const uint4 w = *reinterpret_cast<const uint4*>(ks + sw128<BC>(c, part * DP + 8 * u));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&ww[h]);
          kv[8 * u + 2 * h] = __low2float(pr);
          kv[8 * u + 2 * h + 1] = __high2float(pr);
        }
      }
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const float4* qr = reinterpret_cast<const float4*>(&qs[r * QSTR + part * QP]);
        uint64_t a2 = ssa::f2_pack(0.f, 0.f);
#pragma unroll
        for (int e4 = 0; e4 < DP / 4; ++e4) {
          const float4 qv = qr[e4];
          a2 = ssa::ffma2(ssa::f2_pack(qv.x, qv.y), ssa::f2_pack(kv[4 * e4], kv[4 * e4 + 1]), a2);
          a2 = ssa::ffma2(ssa::f2_pack(qv.z, qv.w), ssa::f2_pack(kv[4 * e4 + 2], kv[4 * e4 + 3]), a2);
        }
        float lo, hi;
        ssa::f2_unpack(a2, lo, hi);
        float acc = lo + hi;
#pragma unroll
        for (int o = 1; o < TPK; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (part == 0) {
          bool vis = (r < R) && (j < p.Lk);
          if (p.causal && r < R) vis = vis && (j <= r % Lq + p.Lk - Lq);
          ss[r * BC + c] = vis ? acc : -INFINITY;
        }
      }
    }
    compute_sync();
    // ---- tile row max and "negligible" per row
#pragma unroll
    for (int u = 0; u < (RT + 7) / 8; ++u) {
      const int r = warp + 8 * u;
      if (r < RT) {
        float mx = -INFINITY;
#pragma unroll
        for (int q4 = 0; q4 < BC / 32; ++q4) mx = fmaxf(mx, ss[r * BC + lane + 32 * q4]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mr = m_run[u];
        const bool neg = (r >= R) || mx == -INFINITY || (mr != -INFINITY && (mx - mr) < p.log2_lambda);
        if (lane == 0) {
          mt_s[r] = mx;
          neg_s[r] = neg ? 1 : 0;
        }
      }
    }
    compute_sync();
    // ---- the vote, one decision per query head
    if (tid < G) {
      int all_neg = 1;
      for (int i = 0; i < Lq; ++i) all_neg &= neg_s[tid * Lq + i];
      keep_s[tid] = !all_neg;
      if (all_neg) ++skipped_tiles;
    }
    compute_sync();
    if (tid == 0) {
      int any = 0;
      for (int g = 0; g < G; ++g) any |= keep_s[g];
      any_keep_s = any;
    }
    // ---- P for the rows of kept heads
#pragma unroll
    for (int u = 0; u < (RT + 7) / 8; ++u) {
      const int r = warp + 8 * u;
      if (r < RT) {
        const bool keep = r < R && keep_s[r / Lq];
        float a = 1.f;
        if (keep) {
          const float mr = m_run[u];
          const float mn = fmaxf(mr, mt_s[r]);
          a = (mr == -INFINITY) ? 0.f : ex2(mr - mn);
          const float mref = (mn == -INFINITY) ? 0.f : mn;
          float sum = 0.f;
#pragma unroll
          for (int q4 = 0; q4 < BC / 32; ++q4) {
            const int c = lane + 32 * q4;
            const float pv = ex2(ss[r * BC + c] - mref);
            ss[r * BC + c] = pv;
            sum += pv;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          l_run[u] = l_run[u] * a + sum;
          m_run[u] = mn;
        } else {
          // a head that skips this tile (or a padding row) adds nothing
#pragma unroll
          for (int q4 = 0; q4 < BC / 32; ++q4) ss[r * BC + lane + 32 * q4] = 0.f;
        }
        if (lane == 0) alpha_s[r] = keep ? a : 1.f;
      }
    }
    compute_sync();
    // ---- O += P V over the kept heads' rows (nothing when no head keeps the tile)
    if (any_keep_s) {
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const float a = alpha_s[r];
        o0[r] *= a;
        o1[r] *= a;
      }
#pragma unroll 4
      for (int c = kg; c < BC; c += NKG) {
        const __nv_bfloat162 vv = *reinterpret_cast<const __nv_bfloat162*>(vs + sw128<BC>(c, 2 * dpair));
        const float v0 = __low2float(vv), v1 = __high2float(vv);  // zeros past Lk (TMA fill), and P = 0 there
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const float pr = ss[r * BC + c];
          o0[r] = fmaf(pr, v0, o0[r]);
          o1[r] = fmaf(pr, v1, o1[r]);
        }
      }
    }
    // the stage's K and V are no longer read: hand it back to the producer
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
    compute_sync();
  }

  // ---- end of the split: sum the P.V partials over key groups, write out
  float* ob = qs;  // RT * D floats (qs holds RT * QSTR >= RT * D)
  for (int e = tid; e < RT * D; e += NTC) ob[e] = 0.f;
  compute_sync();
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    if (r < R) {
      atomicAdd(&ob[r * D + 2 * dpair], o0[r]);
      atomicAdd(&ob[r * D + 2 * dpair + 1], o1[r]);
    }
  }
  compute_sync();
  for (int e = tid; e < R * D; e += NTC) {
    const int r = e / D, dd = e % D;
    const int g = r / Lq, i = r % Lq;
    const int hq = hkv * G + g;
    p.o_part[((((size_t)b * p.Hq + hq) * Lq + i) * p.S + s) * D + dd] = ob[e];
  }
#pragma unroll
  for (int u = 0; u < (RT + 7) / 8; ++u) {
    const int r = warp + 8 * u;
    if (r < R && lane == 0) {
      const int g = r / Lq, i = r % Lq;
      const int hq = hkv * G + g;
      float* ml = p.ml_part + ((((size_t)b * p.Hq + hq) * Lq + i) * p.S + s) * 2;
      ml[0] = m_run[u];
      ml[1] = l_run[u];
    }
  }
  if (tid < G) p.sk_part[((size_t)b * p.Hq + hkv * G + tid) * p.S + s] = skipped_tiles;
}

// Merge the splits of one (batch, head, query row): block of d/2 threads.
template <int D>
__global__ void decode_combine_kernel(const Params p) {
  const int i = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x;  // column pair
  const size_t row = ((size_t)b * p.Hq + hq) * p.Lq + i;
  const float* ml = p.ml_part + row * p.S * 2;
  float M = -INFINITY;
  for (int s = 0; s < p.S; ++s)
    if (ml[2 * s + 1] > 0.f) M = fmaxf(M, ml[2 * s]);
  float L = 0.f, a0 = 0.f, a1 = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.S; ++s) {
      const float ls = ml[2 * s + 1];
      if (!(ls > 0.f)) continue;
      const float w = ex2(ml[2 * s] - M);
      L += w * ls;
      const float* o = p.o_part + (row * p.S + s) * D;
      a0 = fmaf(w, o[2 * t], a0);
      a1 = fmaf(w, o[2 * t + 1], a1);
    }
  }
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

template <int D, int BC, int RT>
static int launch_rt(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, cudaStream_t st) {
  using L = DecSmem<D, BC>;
  const size_t smem = 1024 + L::RING_BYTES + (size_t)RT * ((NTC / BC) * (D / (NTC / BC) + 4) + BC) * 4;
  static bool attr_set[64] = {};  // per instance and device, before the first launch there
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SSA_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(decode_split_kernel<D, BC, RT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return SSA_ERR_CUDA;
    attr_set[dev] = true;
  }
  decode_split_kernel<D, BC, RT><<<dim3(p.S, p.Hkv, p.B), NT, smem, st>>>(mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return SSA_ERR_CUDA;
  decode_combine_kernel<D><<<dim3(p.Lq, p.Hq, p.B), D / 2, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

template <int D, int BC>
static int launch_bc(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, cudaStream_t st) {
  if (p.R <= 4) return launch_rt<D, BC, 4>(mk, mv, p, st);
  if (p.R <= 8) return launch_rt<D, BC, 8>(mk, mv, p, st);
  if (p.R <= 16) return launch_rt<D, BC, 16>(mk, mv, p, st);
  return launch_rt<D, BC, 32>(mk, mv, p, st);
}

static size_t workspace_bytes(int B, int Hq, int Lq, int d, int S) {
  const size_t rows = (size_t)B * Hq * Lq;
  return rows * S * d * sizeof(float) + rows * S * 2 * sizeof(float) + (size_t)B * Hq * S * sizeof(int32_t);
}

}  // namespace ssa_dec

extern "C" {

size_t ssa_decode_workspace_bytes(int B, int Hq, int Lq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || Lq <= 0 || d <= 0 || num_splits <= 0) return 0;
  return ssa_dec::workspace_bytes(B, Hq, Lq, d, num_splits);
}

int ssa_decode(const void* q, const void* k, const void* v, void* out, float* lse,
               int32_t* tile_skip_count, int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal,
               float scale, float lambda, int Bc, int num_splits, void* workspace,
               size_t workspace_bytes, void* stream) {
  using namespace ssa_dec;
  if (!q || !k || !v || !out || !lse || !tile_skip_count || !workspace) return SSA_ERR_INVALID_ARG;
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
  const size_t rows = (size_t)B * Hq * Lq;
  p.o_part = static_cast<float*>(workspace);
  p.ml_part = p.o_part + rows * num_splits * d;
  p.sk_part = reinterpret_cast<int32_t*>(p.ml_part + rows * num_splits * 2);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lk = Lk;
  p.causal = causal ? 1 : 0;
  p.S = num_splits;
  p.nK = (Lk + Bc - 1) / Bc;
  p.tiles_per_split = (p.nK + num_splits - 1) / num_splits;
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

}  // extern "C"
