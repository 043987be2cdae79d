/*
 * ssa_oracle.c -- plain, slow CPU oracle for the skip-softmax / N:M sparse
 * flash-attention forward.  TEST INFRASTRUCTURE ONLY: nothing on the product
 * path may link or call this file; only the tests, the smoke check and the
 * bench's CPU-baseline leg do.  It shares no code with the CUDA kernels.
 *
 * What it computes, in fp64, one (batch b, query head hq, query tile qt) work
 * item at a time, walking key tiles in ascending order exactly as the method
 * describes:
 *
 *   - "Skip-Softmax Sparse Attention for Diffusion Models" (Model-Optimizer,
 *     examples/diffusers/sparsity README, intro paragraph): skip-softmax skips
 *     KV tiles whose attention scores are negligible during the FlashAttention
 *     computation.  Table "Threshold Modes": the kernel compares against the
 *     lambda threshold in the log2 domain.  The exact inequality is the one the
 *     method statement gives: a (Br x Bc) tile is skipped when, for every query
 *     row, exp(tile_row_max - running_max) < lambda.  Skipped tiles change
 *     neither the running max, the running sum nor the accumulator.
 *   - "Attention Sparsity for HuggingFace Models" (Model-Optimizer,
 *     examples/llm_sparsity/attention_sparsity README, "N:M Sparse Softmax"
 *     and the custom N:M configuration): for every M consecutive key positions
 *     keep the top-N scores and set the rest to -inf before softmax; the first
 *     dense_sink_tokens keys and a local window of dense_recent_tokens keys are
 *     excluded from N:M and kept dense.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes):
 *   R1 skip test is strict '<' on natural exp; m is the running max over the
 *      tiles kept so far (before this tile); the first visited tile of a work
 *      item is never skipped unless every row of it is fully masked.
 *   R2 rows whose tile max is -inf (all keys masked in this tile) count as
 *      negligible; rows past Lq do not exist and so never block a skip.
 *   R3 causal masking is bottom-right aligned: query row i sits at key
 *      position pos_i = i + (Lk - Lq) and sees keys j <= pos_i.  Key tiles that
 *      lie wholly above the diagonal are not visited and not counted.
 *   R4 GQA: query head hq reads KV head hq / (Hq / Hkv).
 *   R5 N:M groups are aligned to key index 0: group g = [g*M, g*M + M).  The
 *      top-N ranking runs over the whole group (masked keys rank as -inf,
 *      equal scores rank the lower index first); a key is kept if it is
 *      visible and (in the sink, in the query-relative recent window
 *      0 <= pos_i - j < recent, or ranked < N).  The ranking compares scores
 *      rounded to fp32, the precision the kernel decides in.
 *   R6 N:M masking comes before the tile max and the skip test (combined mode).
 *   R7 a row with no kept key at all gets out = 0 and lse = -inf.
 *   R8 lse is the natural-log log-sum-exp of the scaled scores of kept keys.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SSA_MODE_SKIP 1
#define SSA_MODE_NM 2

typedef struct {
  const uint16_t *q, *k, *v; /* bf16 bit patterns, [B,Lq,Hq,d] and [B,Lk,Hkv,d] */
  int B, Hq, Hkv, Lq, Lk, d, causal;
  double scale;
  int mode;
  double lambda;
  int n, m, sink, recent, Br, Bc;
  double tie_tol;
  const int32_t *items; /* [n_items][3] = (b, hq, qt) */
  int n_items;
  double *out;          /* [n_items][Br][d] */
  double *lse;          /* [n_items][Br] */
  int32_t *skip_count;  /* [n_items] */
  int32_t *visited;     /* [n_items] */
  uint32_t *skip_bits;  /* [n_items][nKw] or NULL: bit kt = tile kt visited and skipped */
  uint32_t *marginal_bits; /* [n_items][nKw] or NULL: bit kt = the tile's largest row ratio within 1e-3*lambda of lambda */
  uint32_t *keep_bits;  /* [n_items][Br][Lkw] or NULL: bit j = key j kept for this row */
  uint32_t *tie_bits;   /* [n_items][Br][Lkw] or NULL: bit j = key j's N:M fate is a near tie */
  const uint32_t *flip_bits; /* [n_items][nKw] or NULL: bit kt = take the other decision (marginal tiles only) */
  int bad_flip;         /* set when flip_bits names a tile that is not marginal */
  int next_item;
  pthread_mutex_t lock;
} job_t;

/* bf16 -> double, exact: a bf16 is the top half of an fp32. */
static double bf16_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static void set_bit(uint32_t *words, long idx) { words[idx >> 5] |= 1u << (idx & 31); }
static int get_bit(const uint32_t *words, long idx) { return (words[idx >> 5] >> (idx & 31)) & 1u; }

/* Number of visited key tiles for a query tile (reading R3). */
static int visited_tiles(int causal, int Lq, int Lk, int Br, int Bc, int qt) {
  int nK = (Lk + Bc - 1) / Bc;
  if (!causal) return nK;
  int last_row = qt * Br + Br - 1;
  if (last_row > Lq - 1) last_row = Lq - 1;
  long last_pos = (long)last_row + (long)(Lk - Lq);
  if (last_pos < 0) return 0;
  long t = last_pos / Bc + 1;
  return t > nK ? nK : (int)t;
}

/* Rank of key j inside its N:M group: how many keys beat it (higher fp32
 * score, or an equal score at a lower index).  Keys outside [0, Lk) or masked
 * carry -inf (reading R5). */
static int group_rank(const float *x32, int g0, int M, int j) {
  int r = 0;
  for (int t = g0; t < g0 + M; ++t) {
    if (t == j) continue;
    if (x32[t - g0] > x32[j - g0] || (x32[t - g0] == x32[j - g0] && t < j)) ++r;
  }
  return r;
}

static void run_item(const job_t *J, int it) {
  const int d = J->d, Br = J->Br, Bc = J->Bc, Lq = J->Lq, Lk = J->Lk;
  const int b = J->items[3 * it + 0], hq = J->items[3 * it + 1], qt = J->items[3 * it + 2];
  const int hkv = hq / (J->Hq / J->Hkv); /* reading R4 */
  const int nK = (Lk + Bc - 1) / Bc, nKw = (nK + 31) / 32, Lkw = (Lk + 31) / 32;
  const int nvis = visited_tiles(J->causal, Lq, Lk, Br, Bc, qt);
  const int skip_on = (J->mode & SSA_MODE_SKIP) != 0, nm_on = (J->mode & SSA_MODE_NM) != 0;
  const int M = J->m, N = J->n;
  const double NEG_INF = -INFINITY;

  int r0 = qt * Br, r1 = qt * Br + Br;
  if (r1 > Lq) r1 = Lq;
  const int rows = r1 - r0 > 0 ? r1 - r0 : 0;

  double *qrow = malloc(sizeof(double) * (size_t)Br * d);
  double *m_run = malloc(sizeof(double) * Br), *l_run = malloc(sizeof(double) * Br);
  double *acc = calloc((size_t)Br * d, sizeof(double));
  double *x = malloc(sizeof(double) * (size_t)Br * Bc);   /* raw q.k of the tile */
  int *kept = malloc(sizeof(int) * (size_t)Br * Bc);      /* visible and kept by N:M */
  double *kd = malloc(sizeof(double) * (size_t)Bc * d), *vd = malloc(sizeof(double) * (size_t)Bc * d);
  double *tmax = malloc(sizeof(double) * Br);

  for (int r = 0; r < rows; ++r) {
    const uint16_t *src = J->q + (((size_t)b * Lq + (r0 + r)) * J->Hq + hq) * d;
    for (int c = 0; c < d; ++c) qrow[(size_t)r * d + c] = bf16_to_double(src[c]);
    m_run[r] = NEG_INF;
    l_run[r] = 0.0;
  }
  int skipped = 0;

  for (int kt = 0; kt < nvis; ++kt) {
    const int c0 = kt * Bc;
    int c1 = c0 + Bc;
    if (c1 > Lk) c1 = Lk;
    const int cols = c1 - c0;
    for (int j = 0; j < cols; ++j) {
      const uint16_t *ks = J->k + (((size_t)b * Lk + (c0 + j)) * J->Hkv + hkv) * d;
      const uint16_t *vs = J->v + (((size_t)b * Lk + (c0 + j)) * J->Hkv + hkv) * d;
      for (int c = 0; c < d; ++c) {
        kd[(size_t)j * d + c] = bf16_to_double(ks[c]);
        vd[(size_t)j * d + c] = bf16_to_double(vs[c]);
      }
    }
    /* scores and masks */
    for (int r = 0; r < rows; ++r) {
      const long pos = (long)(r0 + r) + (long)(Lk - Lq);
      for (int j = 0; j < cols; ++j) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += qrow[(size_t)r * d + c] * kd[(size_t)j * d + c];
        x[(size_t)r * Bc + j] = s;
        kept[(size_t)r * Bc + j] = !(J->causal && (long)(c0 + j) > pos);
      }
    }
    /* N:M selection (readings R5, R6).  Bc is a multiple of M, so a group
     * never straddles two tiles. */
    if (nm_on) {
      float gx[8];
      for (int r = 0; r < rows; ++r) {
        const long pos = (long)(r0 + r) + (long)(Lk - Lq);
        for (int g0 = c0; g0 < c0 + Bc; g0 += M) {
          for (int t = 0; t < M; ++t) {
            const int j = g0 + t;
            gx[t] = (j < Lk && kept[(size_t)r * Bc + (j - c0)]) ? (float)x[(size_t)r * Bc + (j - c0)]
                                                                : -INFINITY;
          }
          /* near-tie detection: the N-th and (N+1)-th largest fp32 scores */
          float srt[8];
          memcpy(srt, gx, sizeof(float) * M);
          for (int a = 1; a < M; ++a) /* insertion sort, descending */
            for (int c = a; c > 0 && srt[c] > srt[c - 1]; --c) {
              float tmp = srt[c]; srt[c] = srt[c - 1]; srt[c - 1] = tmp;
            }
          const int ambiguous =
              N < M && isfinite(srt[N]) && (double)srt[N - 1] - (double)srt[N] <=
                                               J->tie_tol * (1.0 + fabs((double)srt[N - 1]));
          for (int t = 0; t < M; ++t) {
            const int j = g0 + t;
            if (j >= Lk) break;
            int *kp = &kept[(size_t)r * Bc + (j - c0)];
            if (!*kp) continue;
            const int in_window = (j < J->sink) || (pos - j >= 0 && pos - j < J->recent);
            const int top = group_rank(gx, g0, M, j) < N;
            *kp = in_window || top;
            if (J->tie_bits && ambiguous && !in_window) {
              const double gap = fabs((double)gx[t] - (double)srt[N - 1]);
              const double gap2 = fabs((double)gx[t] - (double)srt[N]);
              const double tol = J->tie_tol * (1.0 + fabs((double)srt[N - 1]));
              if (gap <= tol || gap2 <= tol)
                set_bit(J->tie_bits, ((long)it * Br + r) * Lkw * 32 + j);
            }
          }
        }
      }
    }
    /* tile row max over kept keys, in scaled units */
    for (int r = 0; r < rows; ++r) {
      double mx = NEG_INF;
      for (int j = 0; j < cols; ++j)
        if (kept[(size_t)r * Bc + j]) {
          const double s = J->scale * x[(size_t)r * Bc + j];
          if (s > mx) mx = s;
        }
      tmax[r] = mx;
      if (J->keep_bits)
        for (int j = 0; j < cols; ++j)
          if (kept[(size_t)r * Bc + j]) set_bit(J->keep_bits, ((long)it * Br + r) * Lkw * 32 + c0 + j);
    }
    /* skip test (readings R1, R2).  The tile is skipped iff its largest row
     * ratio exp(tmax - m) is below lambda: that largest ratio is the tile's
     * margin quantity, and the tile is "marginal" when it lies within
     * 1e-3 * lambda of lambda (the method statement's tolerance band).  A row
     * with no key in this tile has ratio 0; a row with no kept key yet and a
     * key here has ratio +inf (never negligible, never marginal). */
    if (skip_on) {
      int all_negligible = 1;
      double max_ratio = 0.0;
      for (int r = 0; r < rows; ++r) {
        double ratio;
        if (tmax[r] == NEG_INF) ratio = 0.0;
        else if (m_run[r] == NEG_INF) ratio = INFINITY;
        else ratio = exp(tmax[r] - m_run[r]);
        if (!(ratio < J->lambda)) all_negligible = 0;
        if (ratio > max_ratio) max_ratio = ratio;
      }
      const int marginal = isfinite(max_ratio) && fabs(max_ratio - J->lambda) < 1e-3 * J->lambda;
      if (marginal && J->marginal_bits) set_bit(J->marginal_bits, (long)it * nKw * 32 + kt);
      /* Inside the tolerance band either decision is accepted; a caller that
       * compares against a kernel which took the other one asks for it here
       * (anywhere else the request is an error). */
      if (J->flip_bits && get_bit(J->flip_bits, (long)it * nKw * 32 + kt)) {
        if (!marginal) ((job_t *)J)->bad_flip = 1;
        all_negligible = !all_negligible;
      }
      if (all_negligible) {
        ++skipped;
        if (J->skip_bits) set_bit(J->skip_bits, (long)it * nKw * 32 + kt);
        continue;
      }
    }
    /* online softmax update over the kept keys */
    for (int r = 0; r < rows; ++r) {
      const double m_new = tmax[r] > m_run[r] ? tmax[r] : m_run[r];
      if (m_new == NEG_INF) continue; /* nothing kept yet for this row */
      const double alpha = (m_run[r] == NEG_INF) ? 0.0 : exp(m_run[r] - m_new);
      l_run[r] *= alpha;
      for (int c = 0; c < d; ++c) acc[(size_t)r * d + c] *= alpha;
      for (int j = 0; j < cols; ++j) {
        if (!kept[(size_t)r * Bc + j]) continue;
        const double p = exp(J->scale * x[(size_t)r * Bc + j] - m_new);
        l_run[r] += p;
        for (int c = 0; c < d; ++c) acc[(size_t)r * d + c] += p * vd[(size_t)j * d + c];
      }
      m_run[r] = m_new;
    }
  }

  for (int r = 0; r < Br; ++r) {
    double *o = J->out + ((size_t)it * Br + r) * d;
    if (r < rows && l_run[r] > 0.0) {
      for (int c = 0; c < d; ++c) o[c] = acc[(size_t)r * d + c] / l_run[r];
      J->lse[(size_t)it * Br + r] = m_run[r] + log(l_run[r]);
    } else { /* reading R7, and padding rows past Lq */
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      J->lse[(size_t)it * Br + r] = NEG_INF;
    }
  }
  J->skip_count[it] = skipped;
  J->visited[it] = nvis;

  free(qrow); free(m_run); free(l_run); free(acc); free(x); free(kept);
  free(kd); free(vd); free(tmax);
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  for (;;) {
    pthread_mutex_lock(&J->lock);
    const int it = J->next_item++;
    pthread_mutex_unlock(&J->lock);
    if (it >= J->n_items) break;
    run_item(J, it);
  }
  return NULL;
}

/* Entry point.  Returns 0, -1 on an argument it cannot evaluate, or -2 when
 * flip_bits asks for the other decision on a tile that is not marginal.
 * Output bit arrays must be zeroed by the caller.  Work items are independent, so
 * they are spread over nthreads threads; each item's arithmetic is serial. */
int ssa_oracle_items(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int Hq, int Hkv,
                     int Lq, int Lk, int d, int causal, double scale, int mode, double lambda, int n,
                     int m, int sink, int recent, int Br, int Bc, double tie_tol,
                     const int32_t *items, int n_items, double *out, double *lse,
                     int32_t *skip_count, int32_t *visited, uint32_t *skip_bits,
                     uint32_t *marginal_bits, uint32_t *keep_bits, uint32_t *tie_bits,
                     const uint32_t *flip_bits, int nthreads) {
  if (!q || !k || !v || !items || !out || !lse || !skip_count || !visited) return -1;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lq <= 0 || Lk <= 0 || d <= 0 || Br <= 0 || Bc <= 0)
    return -1;
  if ((mode & SSA_MODE_NM) && (m < 1 || m > 8 || n < 1 || n > m || Bc % m)) return -1;
  for (int i = 0; i < n_items; ++i) {
    const int32_t *w = items + 3 * i;
    if (w[0] < 0 || w[0] >= B || w[1] < 0 || w[1] >= Hq || w[2] < 0 || (long)w[2] * Br >= Lq)
      return -1;
  }
  job_t J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v;
  J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Lq = Lq; J.Lk = Lk; J.d = d; J.causal = causal;
  J.scale = scale; J.mode = mode; J.lambda = lambda; J.n = n; J.m = m;
  J.sink = sink; J.recent = recent; J.Br = Br; J.Bc = Bc; J.tie_tol = tie_tol;
  J.items = items; J.n_items = n_items; J.out = out; J.lse = lse;
  J.skip_count = skip_count; J.visited = visited; J.skip_bits = skip_bits;
  J.marginal_bits = marginal_bits; J.keep_bits = keep_bits; J.tie_bits = tie_bits;
  J.flip_bits = flip_bits;
  pthread_mutex_init(&J.lock, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  int started = 0;
  for (int t = 0; t < nthreads; ++t)
    if (pthread_create(&th[t], NULL, worker, &J) == 0) ++started;
  if (started == 0) worker(&J);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&J.lock);
  return J.bad_flip ? -2 : 0;
}

/* Visited key tiles of one query tile, exported so tests can pin reading R3. */
int ssa_oracle_visited_tiles(int causal, int Lq, int Lk, int Br, int Bc, int qt) {
  return visited_tiles(causal, Lq, Lk, Br, Bc, qt);
}
