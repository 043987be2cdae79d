// ssa_decode.cu -- skip-softmax attention for decode (a few query rows per
// sequence against a long KV cache) on B200 (sm_100a), split over the keys.
//
// Method: "Skip-Softmax Sparse Attention for Diffusion Models" (intro,
// "Threshold Modes") and "Attention Sparsity for HuggingFace Models" (custom
// configuration: per-phase thresholds, prefill and decode; N:M applies to
// prefill only, so this path has no N:M).  A key tile is skipped for a query
// tile when exp(tile_row_max - running_max) < lambda for every row.
//
// Decode is bound by reading the KV cache once, so this path runs on the CUDA
// cores and spreads each sequence's key tiles over `num_splits` CTAs per KV
// head.  Every split runs the skip-softmax recurrence over its own key tiles
// in order, with its own running max (its first tile is never skipped unless
// fully masked); a second kernel merges the splits' (max, sum, accumulator)
// with the usual log-sum-exp rule.  With one split this is exactly the
// prefill rule for a single query tile.
//
// CTA (split s, KV head, batch): the G = Hq / Hkv query heads that share the
// KV head, Lq rows each, R = G * Lq <= 32 rows in all; a key tile is decided
// per query head (its Lq rows), and the V tile is read only if some head
// keeps it.  256 threads:
//   scores  thread t: key t / TPK of the tile, a 1/TPK slice of d; K read
//           straight from global memory (each key row is contiguous), q.k
//           against all R rows, slices combined by shuffles
//   softmax warp w owns rows w, w + 8, ...: tile row max, vote, P, row sum
//   P.V     thread t: two output columns, every (256 / (d/2))-th key of the
//           tile; partial accumulators of all R rows in registers, summed
//           over threads through shared memory at the end of the split
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/ssa.h"

namespace ssa_dec {

constexpr int NT = 256;
constexpr int RMAX = 32;

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* out;
  float* lse;
  int32_t* skip_count;
  float* o_part;    // [B, Hq, Lq, S, d]
  float* ml_part;   // [B, Hq, Lq, S, 2]: running max (log2 units), row sum
  int32_t* sk_part; // [B, Hq, S]
  int B, Hq, Hkv, Lq, Lk, causal, S, nK, tiles_per_split, G, R;
  float c;            // scale * log2(e)
  float log2_lambda;  // -inf for lambda == 0
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int BC, int RT>
__global__ void __launch_bounds__(NT, RT <= 8 ? 2 : 1) decode_split_kernel(const Params p) {
  constexpr int TPK = NT / BC;       // threads per key in the score phase
  constexpr int DP = D / TPK;        // d slice per thread
  constexpr int NDP = D / 2;         // column pairs
  constexpr int NKG = NT / NDP;      // key groups in the P.V phase
  __shared__ __align__(16) float qs[RT * D];   // q * scale * log2 e; reused for the O reduction
  __shared__ __align__(16) float ss[RT * BC];  // scores, then P
  __shared__ float alpha_s[RT];
  __shared__ float mt_s[RT];
  __shared__ int neg_s[RT];
  __shared__ int keep_s[RMAX];  // per query head
  __shared__ int any_keep_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int G = p.G, R = p.R, Lq = p.Lq;
  const int kt0 = s * p.tiles_per_split;
  const int kt1 = min(p.nK, kt0 + p.tiles_per_split);

  // q rows: r = g * Lq + i -> head hkv * G + g, query row i
  for (int e = tid; e < RT * D; e += NT) {
    const int r = e / D, dd = e % D;
    float val = 0.f;
    if (r < R) {
      const int g = r / Lq, i = r % Lq;
      val = __bfloat162float(p.q[(((size_t)b * Lq + i) * p.Hq + hkv * G + g) * D + dd]) * p.c;
    }
    qs[e] = val;
  }
  // per-row state, owned by warp r % 8 (every lane holds a copy)
  float m_run[RT / 8 > 0 ? RT / 8 : 1], l_run[RT / 8 > 0 ? RT / 8 : 1];
#pragma unroll
  for (int u = 0; u < (RT / 8 > 0 ? RT / 8 : 1); ++u) {
    m_run[u] = -INFINITY;
    l_run[u] = 0.f;
  }
  // P.V accumulators: rows 0..RT-1, columns dd, dd + 1 of this thread's pair
  const int dpair = tid % NDP, kg = tid / NDP;
  float o0[RT], o1[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) o0[r] = o1[r] = 0.f;
  int skipped_tiles = 0;  // per head, kept by thread g (< G)
  __syncthreads();

  const size_t kv_row = (size_t)p.Hkv * D;  // elements between consecutive keys
  const __nv_bfloat16* kbase = p.k + ((size_t)b * p.Lk * p.Hkv + hkv) * D;
  const __nv_bfloat16* vbase = p.v + ((size_t)b * p.Lk * p.Hkv + hkv) * D;

  // this thread's slice of key tile kt's K, raw bf16 (zeros past Lk); the next
  // tile's slice is loaded while the current tile's P.V runs
  const int kc = tid / TPK, kpart = tid % TPK;
  uint4 kraw[DP / 8];
  auto load_k = [&](int kt) {
    const int j = kt * BC + kc;
    if (kt < kt1 && j < p.Lk) {
      const uint4* src = reinterpret_cast<const uint4*>(kbase + (size_t)j * kv_row + kpart * DP);
#pragma unroll
      for (int u = 0; u < DP / 8; ++u) kraw[u] = src[u];
    } else {
#pragma unroll
      for (int u = 0; u < DP / 8; ++u) kraw[u] = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  load_k(kt0);

  // V pairs of the current tile; issued before the tile's scores when the
  // previous tile was kept (so their latency hides behind the softmax), else
  // only once the vote has kept this tile
  constexpr int NV = BC / NKG;
  uint32_t vraw[NV];
  auto load_v = [&](int j0) {
    const int ncols = min(BC, p.Lk - j0);
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      const int c = kg + NKG * u;
      vraw[u] = c < ncols ? *reinterpret_cast<const uint32_t*>(vbase + (size_t)(j0 + c) * kv_row + 2 * dpair)
                          : 0u;
    }
  };
  bool prev_any_keep = true;

  for (int kt = kt0; kt < kt1; ++kt) {
    const int j0 = kt * BC;
    const bool v_early = prev_any_keep;
    if (v_early) load_v(j0);
    // ---- scores: ss[r][c] = q_r . k_{j0+c} in log2 units (-inf where masked)
    {
      const int c = kc, part = kpart;
      const int j = j0 + c;
      float kv[DP];
#pragma unroll
      for (int u = 0; u < DP / 8; ++u) {
        const uint32_t ww[4] = {kraw[u].x, kraw[u].y, kraw[u].z, kraw[u].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&ww[h]);
          kv[8 * u + 2 * h] = __low2float(pr);
          kv[8 * u + 2 * h + 1] = __high2float(pr);
        }
      }
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const float* qr = &qs[r * D + part * DP];
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < DP; ++e) acc = fmaf(qr[e], kv[e], acc);
#pragma unroll
        for (int o = 1; o < TPK; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (part == 0) {
          bool vis = (r < R) && (j < p.Lk);
          if (p.causal && r < R) vis = vis && (j <= r % Lq + p.Lk - Lq);
          ss[r * BC + c] = vis ? acc : -INFINITY;
        }
      }
    }
    // the next tile's K is on its way during the rest of this tile
    load_k(kt + 1);
    __syncthreads();
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
        const bool neg = (r >= R) || mx == -INFINITY ||
                         (mr != -INFINITY && (mx - mr) < p.log2_lambda);
        if (lane == 0) {
          mt_s[r] = mx;
          neg_s[r] = neg ? 1 : 0;
        }
      }
    }
    __syncthreads();
    // ---- the vote, one decision per query head
    if (tid < G) {
      int all_neg = 1;
      for (int i = 0; i < Lq; ++i) all_neg &= neg_s[tid * Lq + i];
      keep_s[tid] = !all_neg;
      if (all_neg) ++skipped_tiles;
    }
    __syncthreads();
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
    __syncthreads();
    // ---- O += P V over the kept heads' rows; V is not read when no head keeps the
    // tile unless it was requested early (previous tile kept)
    const bool any_keep = any_keep_s != 0;
    prev_any_keep = any_keep;
    if (any_keep) {
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const float a = alpha_s[r];
        o0[r] *= a;
        o1[r] *= a;
      }
      // this thread's V pairs of the tile (columns past Lk read nothing and have P = 0)
      if (!v_early) load_v(j0);
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const int c = kg + NKG * u;
        const __nv_bfloat162 vv = *reinterpret_cast<const __nv_bfloat162*>(&vraw[u]);
        const float v0 = __low2float(vv), v1 = __high2float(vv);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const float pr = ss[r * BC + c];  // 0 for rows of heads that skip the tile
          o0[r] = fmaf(pr, v0, o0[r]);
          o1[r] = fmaf(pr, v1, o1[r]);
        }
      }
    }
    __syncthreads();
  }

  // ---- end of the split: sum the P.V partials over key groups, write out
  float* ob = qs;  // RT * D floats
  for (int e = tid; e < RT * D; e += NT) ob[e] = 0.f;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    if (r < R) {
      atomicAdd(&ob[r * D + 2 * dpair], o0[r]);
      atomicAdd(&ob[r * D + 2 * dpair + 1], o1[r]);
    }
  }
  __syncthreads();
  for (int e = tid; e < R * D; e += NT) {
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
static int launch_rt(const Params& p, cudaStream_t st) {
  decode_split_kernel<D, BC, RT><<<dim3(p.S, p.Hkv, p.B), NT, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SSA_ERR_CUDA;
  decode_combine_kernel<D><<<dim3(p.Lq, p.Hq, p.B), D / 2, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

template <int D, int BC>
static int launch_bc(const Params& p, cudaStream_t st) {
  if (p.R <= 4) return launch_rt<D, BC, 4>(p, st);
  if (p.R <= 8) return launch_rt<D, BC, 8>(p, st);
  if (p.R <= 16) return launch_rt<D, BC, 16>(p, st);
  return launch_rt<D, BC, 32>(p, st);
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
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
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
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128) return Bc == 128 ? launch_bc<128, 128>(p, st) : launch_bc<128, 64>(p, st);
  return Bc == 128 ? launch_bc<64, 128>(p, st) : launch_bc<64, 64>(p, st);
}

}  // extern "C"
