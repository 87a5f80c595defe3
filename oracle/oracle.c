/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the heterogeneous-batch paged
 * LoRA delta.  TEST INFRASTRUCTURE ONLY: nothing in the product path links,
 * loads or calls this file; only the tests, the package's smoke entry and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or helper
 * with the CUDA path.
 *
 * What it computes (each function cites the passage it follows):
 *
 *  oracle_lora_delta   -- y_i <- y_i + (alpha / r_a) * ((x_i . A_a) . B_a) for
 *                         every token i with adapter a = idx[i] >= 0.
 *      * the per-token loop with the "adapter id < 0 means skip" rule is the
 *        Python reference loop of "Paper explainer: S-LoRA" (0h-n0.github.io,
 *        section "BGMV kernel", bgmv_reference);
 *      * the scaled, row-vector form Y = X.W0 + (alpha/r).((X.A).B) and the
 *        order "shrink by A, then expand by B" are from "Multi-LoRA serving:
 *        S-LoRA, Punica, SGMV, vLLM" (produtoramaxvision.com.br), section on
 *        how the SGMV kernel executes concurrent adapters.
 *      The sums are written out in fp64, in ascending index order.  The base
 *      term X.W0 is outside the path: y_in stands for it.
 *      Storage: A is held transposed, r rows of d_in (rank-major); B is r rows
 *      of d_out.  Element values are fp16 or bf16 bit patterns, decoded
 *      exactly to fp64 by the decoders below.
 *
 *  oracle_linear       -- the base term of the same page's scaled form,
 *                         y = X.W0 (W0 stored as d_out rows of d_in, the
 *                         layout of a linear layer's weight), fp64 sums in
 *                         ascending index order.  With oracle_lora_delta it
 *                         gives the whole linear layer with its LoRA delta,
 *                         Y = X.W0 + (alpha/r).((X.A).B) -- the output that the
 *                         "residual add fused into the linear layer's output"
 *                         remark of the page's metrics section refers to.
 *  oracle_segments     -- stable counting sort of tokens by adapter id: the
 *                         segment structure of SGMV ("index vector maps each
 *                         token to its adapter", same SGMV section).
 *  oracle_merge_requests -- contiguous request ranges -> segments, merging
 *                         neighbouring requests that use the same adapter.
 *  oracle_pages_needed -- pages a rank-r adapter occupies when each of its
 *                         tensors is laid out flat over fixed-size pages, so that
 *                         only the last page of each tensor is partly empty
 *                         (same page's section on the unified paged pool).
 *  oracle_decode_e4m3, oracle_quantize_e4m3, oracle_lora_delta_q8 -- the delta
 *                         with 8-bit adapter weights (e4m3, one fp32 scale per
 *                         rank row): "Multi-LoRA serving", trade-offs section
 *                         (adapters quantised to FP8 or INT4 halve their PCIe
 *                         traffic and let more of them stay resident) and SGMV
 *                         section (the segmented kernels exist in FP8 form).  The
 *                         per-row scale is a reading: the page gives none.  Test
 *                         infrastructure ahead of the kernels for that format.
 *  oracle_lru_run      -- least-recently-used residency decisions over a trace
 *                         of page-in calls ("Paper explainer: S-LoRA", section
 *                         "Unified Paging", eviction strategy).
 *  oracle_lru_prefetch_run -- the same with prefetch calls interleaved: adapters
 *                         loaded ahead of the step that uses them, without
 *                         disturbing the current step ("Paper explainer:
 *                         S-LoRA", implementation notes on pre-loading frequent
 *                         adapters; "Multi-LoRA serving", unified pool section:
 *                         the scheduler anticipates requests), and with KV-cache
 *                         blocks taking and returning pages of the same pool
 *                         ("Paper explainer: S-LoRA", section "Unified Paging").
 *
 * Readings where the pages are silent are listed in the design notes; the ones
 * that shape this file: rank 0 leaves y unchanged; ties in LRU age go to the
 * lower adapter id; a page-in call either succeeds whole or changes nothing.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_OOM 2

/* ------------------------------------------------------------------------- */
/* 16-bit float decoding, exact.                                              */
/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.             */
static double dec_f16(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f + 1024), e - 25); /* (1.f) * 2^(e-15) */
  return s ? -v : v;
}
/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. */
static double dec_bf16(uint16_t b) {
  int s = (b >> 15) & 1, e = (b >> 7) & 0xff, f = b & 0x7f;
  double v;
  if (e == 0)
    v = ldexp((double)f, -133); /* f * 2^-126 * 2^-7 */
  else if (e == 255)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f + 128), e - 134); /* (1.f) * 2^(e-127) */
  return s ? -v : v;
}
static double dec(int dtype, uint16_t v) { return dtype == 1 ? dec_bf16(v) : dec_f16(v); }

/* dtype: 0 = fp16, 1 = bf16 */
int oracle_decode16(int dtype, const uint16_t* in, long n, double* out) {
  if (dtype != 0 && dtype != 1) return OR_ERR_ARG;
  for (long i = 0; i < n; ++i) out[i] = dec(dtype, in[i]);
  return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* The delta.                                                                 */
typedef struct {
  int dtype, T, d_in, d_out;
  const uint16_t* x;
  long ldx;
  const int* idx;
  const uint16_t* y_in;
  long ldy;
  int n_adapters;
  const int* rank;
  const double* alpha;
  const uint16_t* const* A_t; /* [adapter] -> rank x d_in   */
  const uint16_t* const* B;   /* [adapter] -> rank x d_out  */
  double* y_out;              /* T x d_out                  */
  int t0, t1;
} delta_job;

static void* delta_worker(void* arg) {
  delta_job* J = (delta_job*)arg;
  double* t = NULL;
  int tcap = 0;
  for (int i = J->t0; i < J->t1; ++i) {
    double* yo = J->y_out + (long)i * J->d_out;
    const uint16_t* yi = J->y_in ? J->y_in + (long)i * J->ldy : NULL;
    for (int l = 0; l < J->d_out; ++l) yo[l] = yi ? dec(J->dtype, yi[l]) : 0.0;
    int a = J->idx[i];
    if (a < 0) continue; /* "adapter id < 0": row untouched */
    int r = J->rank[a];
    if (r == 0) continue; /* rank 0: nothing to add */
    if (r > tcap) {
      free(t);
      t = (double*)malloc(sizeof(double) * r);
      tcap = r;
    }
    const uint16_t* xi = J->x + (long)i * J->ldx;
    const uint16_t* At = J->A_t[a];
    const uint16_t* B = J->B[a];
    /* shrink: t[k] = sum_j x[j] * A[j][k],   A[j][k] = A_t[k][j] */
    for (int k = 0; k < r; ++k) {
      double acc = 0.0;
      for (int j = 0; j < J->d_in; ++j)
        acc += dec(J->dtype, xi[j]) * dec(J->dtype, At[(long)k * J->d_in + j]);
      t[k] = acc;
    }
    /* expand and scale: y[l] += (alpha / r) * sum_k t[k] * B[k][l] */
    double s = J->alpha[a] / (double)r;
    for (int l = 0; l < J->d_out; ++l) {
      double acc = 0.0;
      for (int k = 0; k < r; ++k) acc += t[k] * dec(J->dtype, B[(long)k * J->d_out + l]);
      yo[l] += s * acc;
    }
  }
  free(t);
  return NULL;
}

/*
 * y_out[i][l] (fp64, not rounded) for i < T, l < d_out.  y_in may be NULL
 * (taken as zero).  idx[i] in [-1, n_adapters).  n_threads >= 1 splits the
 * token range; the result does not depend on it.
 */
int oracle_lora_delta(int dtype, int T, int d_in, int d_out, const uint16_t* x, long ldx,
                      const int* idx, const uint16_t* y_in, long ldy, int n_adapters,
                      const int* rank, const double* alpha, const uint16_t* const* A_t,
                      const uint16_t* const* B, double* y_out, int n_threads) {
  if ((dtype != 0 && dtype != 1) || T < 0 || d_in <= 0 || d_out <= 0 || ldx < d_in ||
      (y_in && ldy < d_out) || n_threads < 1)
    return OR_ERR_ARG;
  for (int i = 0; i < T; ++i)
    if (idx[i] < -1 || idx[i] >= n_adapters) return OR_ERR_ARG;
  for (int i = 0; i < T; ++i)
    if (idx[i] >= 0 && (rank[idx[i]] < 0 || (rank[idx[i]] > 0 && (!A_t[idx[i]] || !B[idx[i]]))))
      return OR_ERR_ARG;
  if (n_threads > T) n_threads = T > 0 ? T : 1;
  delta_job* jobs = (delta_job*)calloc(n_threads, sizeof(delta_job));
  pthread_t* th = (pthread_t*)calloc(n_threads, sizeof(pthread_t));
  for (int w = 0; w < n_threads; ++w) {
    delta_job j = {dtype, T, d_in, d_out, x, ldx, idx, y_in, ldy, n_adapters, rank, alpha,
                   A_t, B, y_out, (int)((long)T * w / n_threads),
                   (int)((long)T * (w + 1) / n_threads)};
    jobs[w] = j;
  }
  for (int w = 1; w < n_threads; ++w) pthread_create(&th[w], NULL, delta_worker, &jobs[w]);
  delta_worker(&jobs[0]);
  for (int w = 1; w < n_threads; ++w) pthread_join(th[w], NULL);
  free(jobs);
  free(th);
  return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* Segments.                                                                  */
/*
 * Tokens with idx >= 0, ordered by adapter id ascending and, inside one
 * adapter, by token position (a stable counting sort).  perm[0..n_valid),
 * seg_start[0..S], seg_adapter[0..S).  Tokens with idx == -1 are left out.
 */
int oracle_segments(const int* idx, int T, int max_adapters, int* perm, int* seg_start,
                    int* seg_adapter, int* S_out) {
  if (T < 0 || max_adapters <= 0) return OR_ERR_ARG;
  for (int i = 0; i < T; ++i)
    if (idx[i] < -1 || idx[i] >= max_adapters) return OR_ERR_ARG;
  int* count = (int*)calloc(max_adapters, sizeof(int));
  for (int i = 0; i < T; ++i)
    if (idx[i] >= 0) count[idx[i]]++;
  int* start = (int*)calloc(max_adapters, sizeof(int));
  int pos = 0, S = 0;
  for (int a = 0; a < max_adapters; ++a) {
    start[a] = pos;
    if (count[a] > 0) {
      seg_start[S] = pos;
      seg_adapter[S] = a;
      S++;
    }
    pos += count[a];
  }
  seg_start[S] = pos;
  for (int i = 0; i < T; ++i) /* ascending i keeps the sort stable */
    if (idx[i] >= 0) perm[start[idx[i]]++] = i;
  *S_out = S;
  free(count);
  free(start);
  return OR_OK;
}

/*
 * Prefill: request q covers tokens [req_start[q], req_start[q+1]) and uses
 * adapter req_adapter[q] (-1: none).  Neighbouring requests with the same
 * adapter become one segment; segments partition [req_start[0], req_start[n]).
 * Empty requests are dropped.
 */
int oracle_merge_requests(const int* req_start, const int* req_adapter, int n, int* seg_start,
                          int* seg_adapter, int* S_out) {
  if (n < 0) return OR_ERR_ARG;
  int S = 0;
  for (int q = 0; q < n; ++q) {
    if (req_start[q + 1] < req_start[q] || req_adapter[q] < -1) return OR_ERR_ARG;
    if (req_start[q + 1] == req_start[q]) continue;
    if (S > 0 && seg_adapter[S - 1] == req_adapter[q]) continue; /* extends the open segment */
    seg_start[S] = req_start[q];
    seg_adapter[S] = req_adapter[q];
    S++;
  }
  seg_start[S] = n > 0 ? req_start[n] : 0;
  *S_out = S;
  return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* Pages.                                                                     */
static long cdiv(long a, long b) { return (a + b - 1) / b; }

/* Each of the 2*n_proj tensors (r x d_in for A, r x d_out for B) is laid out
 * flat and cut into pages of page_elems elements. */
long oracle_pages_needed(int rank, int n_proj, const int* d_in, const int* d_out,
                         long page_elems) {
  long n = 0;
  for (int p = 0; p < n_proj; ++p)
    n += cdiv((long)rank * d_in[p], page_elems) + cdiv((long)rank * d_out[p], page_elems);
  return n;
}

/* ------------------------------------------------------------------------- */
/* The base linear map y = x . W0 (W0 given as d_out rows of d_in).          */
typedef struct {
  int dtype, d_in, d_out;
  const uint16_t* x;
  long ldx;
  const uint16_t* w;
  long ldw;
  double* y;
  int t0, t1;
} linear_job;

static void* linear_worker(void* arg) {
  linear_job* J = (linear_job*)arg;
  double* xr = (double*)malloc(sizeof(double) * J->d_in);
  for (int i = J->t0; i < J->t1; ++i) {
    for (int j = 0; j < J->d_in; ++j) xr[j] = dec(J->dtype, J->x[(long)i * J->ldx + j]);
    for (int l = 0; l < J->d_out; ++l) {
      const uint16_t* wl = J->w + (long)l * J->ldw;
      double acc = 0.0;
      for (int j = 0; j < J->d_in; ++j) acc += xr[j] * dec(J->dtype, wl[j]);
      J->y[(long)i * J->d_out + l] = acc;
    }
  }
  free(xr);
  return NULL;
}

int oracle_linear(int dtype, int T, int d_in, int d_out, const uint16_t* x, long ldx, const uint16_t* w,
                  long ldw, double* y_out, int n_threads) {
  if ((dtype != 0 && dtype != 1) || T < 0 || d_in <= 0 || d_out <= 0 || ldx < d_in || ldw < d_in ||
      n_threads < 1)
    return OR_ERR_ARG;
  if (n_threads > T) n_threads = T > 0 ? T : 1;
  linear_job* jobs = (linear_job*)calloc(n_threads, sizeof(linear_job));
  pthread_t* th = (pthread_t*)calloc(n_threads, sizeof(pthread_t));
  for (int k = 0; k < n_threads; ++k) {
    linear_job j = {dtype, d_in, d_out, x, ldx, w, ldw, y_out, (int)((long)T * k / n_threads),
                    (int)((long)T * (k + 1) / n_threads)};
    jobs[k] = j;
  }
  for (int k = 1; k < n_threads; ++k) pthread_create(&th[k], NULL, linear_worker, &jobs[k]);
  linear_worker(&jobs[0]);
  for (int k = 1; k < n_threads; ++k) pthread_join(th[k], NULL);
  free(jobs);
  free(th);
  return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* LRU.                                                                       */
/*
 * A pool of `capacity` pages and adapters 0..n_adapters-1 needing need[a]
 * pages each.  Call c asks for ids[call_off[c] .. call_off[c+1]) (duplicates
 * allowed).  For each call:
 *   - every asked adapter must end up resident; the asked ones are pinned for
 *     this call and cannot be evicted by it;
 *   - while the free pages do not cover the missing adapters, the resident,
 *     unpinned adapter with the oldest last use is evicted (equal ages: the
 *     lower id first); never-used counts as oldest;
 *   - if that cannot make room, the call fails with OOM and nothing changes;
 *   - on success every asked adapter gets last use = c.
 * Missing adapters are loaded in the order they first appear in the call.
 * Outputs: status[c]; resident[c*n_adapters + a] after call c; the evicted ids
 * of all calls concatenated in eviction order, with evict_off[c] marking where
 * call c starts (evict_off has n_calls+1 entries).
 */
int oracle_lru_run(int n_adapters, const long* need, long capacity, int n_calls,
                   const int* call_off, const int* ids, int* status, unsigned char* resident,
                   int* evicted, int* evict_off) {
  unsigned char* res = (unsigned char*)calloc(n_adapters, 1);
  long* last = (long*)malloc(sizeof(long) * n_adapters);
  unsigned char* pin = (unsigned char*)calloc(n_adapters, 1);
  unsigned char* tmp = (unsigned char*)malloc(n_adapters);
  int* victims = (int*)malloc(sizeof(int) * (n_adapters + 1));
  for (int a = 0; a < n_adapters; ++a) last[a] = -1;
  long used = 0;
  int ne = 0;
  for (int c = 0; c < n_calls; ++c) {
    evict_off[c] = ne;
    memset(pin, 0, n_adapters);
    int bad = 0;
    long missing = 0;
    for (int q = call_off[c]; q < call_off[c + 1]; ++q) {
      int a = ids[q];
      if (a < 0 || a >= n_adapters) {
        bad = 1;
        break;
      }
      if (!pin[a] && !res[a]) missing += need[a];
      pin[a] = 1;
    }
    if (bad) {
      status[c] = OR_ERR_ARG;
    } else {
      /* plan evictions without changing state */
      memcpy(tmp, res, n_adapters);
      long free_pages = capacity - used;
      int nv = 0;
      while (free_pages < missing) {
        int best = -1;
        for (int a = 0; a < n_adapters; ++a) {
          if (!tmp[a] || pin[a]) continue;
          if (best < 0 || last[a] < last[best]) best = a; /* ascending a: ties keep lower id */
        }
        if (best < 0) break;
        tmp[best] = 0;
        free_pages += need[best];
        victims[nv++] = best;
      }
      if (free_pages < missing) {
        status[c] = OR_ERR_OOM;
      } else {
        for (int v = 0; v < nv; ++v) {
          res[victims[v]] = 0;
          used -= need[victims[v]];
          evicted[ne++] = victims[v];
        }
        for (int q = call_off[c]; q < call_off[c + 1]; ++q) {
          int a = ids[q];
          if (!res[a]) {
            res[a] = 1;
            used += need[a];
          }
          last[a] = c;
        }
        status[c] = OR_OK;
      }
    }
    memcpy(resident + (long)c * n_adapters, res, n_adapters);
  }
  evict_off[n_calls] = ne;
  free(res);
  free(last);
  free(pin);
  free(tmp);
  free(victims);
  return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* LRU with prefetch.                                                         */
/*
 * As oracle_lru_run, with each call c of kind[c]:
 *   0 (page-in): as above; on success the step counter E grows by one and
 *     every asked adapter gets age E;
 *   1 (prefetch, page budget budget[c]): the asked adapters that are not
 *     resident are taken in the order they first appear; one is chosen when
 *     the pages chosen so far plus its own stay within min(budget[c], free
 *     pages + pages of the resident adapters older than E), else it is
 *     skipped and the next is tried.  Room is made by evicting resident
 *     adapters older than E, oldest first (equal ages: lower id first).  The
 *     chosen adapters become resident with age E.  Status OK unless an id is
 *     out of range (ARG, nothing changes);
 *   2 (KV blocks take budget[c] pages): when the free pages do not cover them,
 *     resident adapters older than E are evicted, oldest first (equal ages:
 *     lower id first); if even all of those cannot make room: OOM, nothing
 *     changes;
 *   3 (KV blocks return budget[c] pages);
 *   4 (explicit eviction of the one adapter ids[call_off[c]]): ARG if it is
 *     out of range, NOT_RESIDENT (3) if it is not resident, else it leaves the
 *     pool (ages and E unchanged).
 * Pages held by KV blocks are neither free nor evictable.
 * Ages start at -1 (never used); E starts at 0.
 */
int oracle_lru_prefetch_run(int n_adapters, const long* need, long capacity, int n_calls,
                            const int* kind, const long* budget, const int* call_off, const int* ids,
                            int* status, unsigned char* resident) {
  unsigned char* res = (unsigned char*)calloc(n_adapters, 1);
  long* age = (long*)malloc(sizeof(long) * n_adapters);
  unsigned char* mark = (unsigned char*)calloc(n_adapters, 1);
  unsigned char* tmp = (unsigned char*)malloc(n_adapters);
  int* order = (int*)malloc(sizeof(int) * (n_adapters + 1));
  for (int a = 0; a < n_adapters; ++a) age[a] = -1;
  long used = 0, kv = 0, E = 0;
  for (int c = 0; c < n_calls; ++c) {
    if (kind[c] == 4) {
      const int a = call_off[c + 1] > call_off[c] ? ids[call_off[c]] : -1;
      if (a < 0 || a >= n_adapters) {
        status[c] = OR_ERR_ARG;
      } else if (!res[a]) {
        status[c] = 3;
      } else {
        res[a] = 0;
        used -= need[a];
        status[c] = OR_OK;
      }
      memcpy(resident + (long)c * n_adapters, res, n_adapters);
      continue;
    }
    if (kind[c] == 2 || kind[c] == 3) {
      if (kind[c] == 3) {
        kv -= budget[c];
        status[c] = OR_OK;
      } else {
        long room = capacity - used - kv;
        for (int a = 0; a < n_adapters; ++a)
          if (res[a] && age[a] < E) room += need[a];
        if (room < budget[c]) {
          status[c] = OR_ERR_OOM;
        } else {
          while (capacity - used - kv < budget[c]) {
            int best = -1;
            for (int a = 0; a < n_adapters; ++a)
              if (res[a] && age[a] < E && (best < 0 || age[a] < age[best])) best = a;
            res[best] = 0;
            used -= need[best];
          }
          kv += budget[c];
          status[c] = OR_OK;
        }
      }
      memcpy(resident + (long)c * n_adapters, res, n_adapters);
      continue;
    }
    int bad = 0;
    for (int q = call_off[c]; q < call_off[c + 1]; ++q)
      if (ids[q] < 0 || ids[q] >= n_adapters) bad = 1;
    memset(mark, 0, n_adapters);
    if (bad) {
      status[c] = OR_ERR_ARG;
    } else if (kind[c] == 0) {
      long missing = 0;
      for (int q = call_off[c]; q < call_off[c + 1]; ++q) {
        int a = ids[q];
        if (!mark[a] && !res[a]) missing += need[a];
        mark[a] = 1; /* pinned for this call */
      }
      memcpy(tmp, res, n_adapters);
      long free_pages = capacity - used - kv;
      while (free_pages < missing) {
        int best = -1;
        for (int a = 0; a < n_adapters; ++a)
          if (tmp[a] && !mark[a] && (best < 0 || age[a] < age[best])) best = a;
        if (best < 0) break;
        tmp[best] = 0;
        free_pages += need[best];
      }
      if (free_pages < missing) {
        status[c] = OR_ERR_OOM;
      } else {
        for (int a = 0; a < n_adapters; ++a)
          if (res[a] && !tmp[a]) {
            res[a] = 0;
            used -= need[a];
          }
        E += 1;
        for (int q = call_off[c]; q < call_off[c + 1]; ++q) {
          int a = ids[q];
          if (!res[a]) {
            res[a] = 1;
            used += need[a];
          }
          age[a] = E;
        }
        status[c] = OR_OK;
      }
    } else {
      long room = capacity - used - kv;
      for (int a = 0; a < n_adapters; ++a)
        if (res[a] && age[a] < E) room += need[a];
      long limit = budget[c] < room ? budget[c] : room;
      long chosen = 0;
      int n_order = 0;
      for (int q = call_off[c]; q < call_off[c + 1]; ++q) {
        int a = ids[q];
        if (res[a] || mark[a]) continue;
        mark[a] = 1; /* looked at (first occurrence decides) */
        if (chosen + need[a] > limit) continue;
        order[n_order++] = a;
        chosen += need[a];
      }
      long free_pages = capacity - used - kv;
      while (free_pages < chosen) {
        int best = -1;
        for (int a = 0; a < n_adapters; ++a)
          if (res[a] && age[a] < E && (best < 0 || age[a] < age[best])) best = a;
        if (best < 0) break; /* cannot happen: chosen <= room */
        res[best] = 0;
        used -= need[best];
        free_pages += need[best];
      }
      for (int k = 0; k < n_order; ++k) {
        res[order[k]] = 1;
        used += need[order[k]];
        age[order[k]] = E;
      }
      status[c] = OR_OK;
    }
    memcpy(resident + (long)c * n_adapters, res, n_adapters);
  }
  free(res);
  free(age);
  free(mark);
  free(tmp);
  free(order);
  return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* 8-bit adapter weights.                                                     */
/* e4m3 in its "fn" form: 1 sign, 4 exponent (bias 7), 3 fraction bits, no
 * infinities; exponent 15 with fraction 7 is NaN; the largest finite value is
 * 448 (exponent 15, fraction 6). */
static double dec_e4m3(uint8_t b) {
  int s = (b >> 7) & 1, e = (b >> 3) & 0xf, f = b & 7;
  double v;
  if (e == 15 && f == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)f, -9); /* subnormal: f * 2^-3 * 2^-6 */
  else
    v = ldexp((double)(f + 8), e - 10); /* (1.f) * 2^(e-7) */
  return s ? -v : v;
}

int oracle_decode_e4m3(const uint8_t* in, long n, double* out) {
  for (long i = 0; i < n; ++i) out[i] = dec_e4m3(in[i]);
  return OR_OK;
}

/* The finite e4m3 value nearest to v, found by trying every non-negative
 * finite code; a tie goes to the code with an even fraction; beyond 448 the
 * result saturates at +-448.  v must not be NaN. */
static uint8_t enc_e4m3(double v) {
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const double a = fabs(v);
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c <= 0x7e; ++c) {
    const double d = fabs(a - dec_e4m3((uint8_t)c));
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return (uint8_t)(sign | best);
}

/* out[i] = the e4m3 code nearest to in[i] / scale (scale > 0), or 0 when
 * scale == 0 (an all-zero row). */
int oracle_quantize_e4m3(const double* in, long n, double scale, uint8_t* out) {
  if (!(scale >= 0)) return OR_ERR_ARG;
  for (long i = 0; i < n; ++i) {
    if (isnan(in[i])) return OR_ERR_ARG;
    out[i] = scale == 0 ? 0 : enc_e4m3(in[i] / scale);
  }
  return OR_OK;
}

typedef struct {
  int dtype, T, d_in, d_out;
  const uint16_t* x;
  long ldx;
  const int* idx;
  const uint16_t* y_in;
  long ldy;
  const int* rank;
  const double* alpha;
  const uint8_t* const* qA; /* [adapter] -> rank x d_in codes  */
  const float* const* sA;   /* [adapter] -> rank row scales    */
  const uint8_t* const* qB; /* [adapter] -> rank x d_out codes */
  const float* const* sB;
  double* y_out;
  int t0, t1;
} q8_job;

static void* q8_worker(void* arg) {
  q8_job* J = (q8_job*)arg;
  double* t = NULL;
  int tcap = 0;
  for (int i = J->t0; i < J->t1; ++i) {
    double* yo = J->y_out + (long)i * J->d_out;
    const uint16_t* yi = J->y_in ? J->y_in + (long)i * J->ldy : NULL;
    for (int l = 0; l < J->d_out; ++l) yo[l] = yi ? dec(J->dtype, yi[l]) : 0.0;
    int a = J->idx[i];
    if (a < 0) continue;
    int r = J->rank[a];
    if (r == 0) continue;
    if (r > tcap) {
      free(t);
      t = (double*)malloc(sizeof(double) * r);
      tcap = r;
    }
    const uint16_t* xi = J->x + (long)i * J->ldx;
    /* shrink: t[k] = sA[k] * sum_j x[j] * qA[k][j] */
    for (int k = 0; k < r; ++k) {
      double acc = 0.0;
      for (int j = 0; j < J->d_in; ++j)
        acc += dec(J->dtype, xi[j]) * dec_e4m3(J->qA[a][(long)k * J->d_in + j]);
      t[k] = (double)J->sA[a][k] * acc;
    }
    /* expand and scale: y[l] += (alpha / r) * sum_k t[k] * (sB[k] * qB[k][l]) */
    double s = J->alpha[a] / (double)r;
    for (int l = 0; l < J->d_out; ++l) {
      double acc = 0.0;
      for (int k = 0; k < r; ++k)
        acc += t[k] * ((double)J->sB[a][k] * dec_e4m3(J->qB[a][(long)k * J->d_out + l]));
      yo[l] += s * acc;
    }
  }
  free(t);
  return NULL;
}

/* As oracle_lora_delta, with adapter a's weights given as e4m3 codes and one
 * fp32 scale per rank row: A[j][k] = sA[k] * e4m3(qA[k][j]) (A held
 * transposed, rank-major), B[k][l] = sB[k] * e4m3(qB[k][l]). */
int oracle_lora_delta_q8(int dtype, int T, int d_in, int d_out, const uint16_t* x, long ldx,
                         const int* idx, const uint16_t* y_in, long ldy, int n_adapters,
                         const int* rank, const double* alpha, const uint8_t* const* qA,
                         const float* const* sA, const uint8_t* const* qB, const float* const* sB,
                         double* y_out, int n_threads) {
  if ((dtype != 0 && dtype != 1) || T < 0 || d_in <= 0 || d_out <= 0 || ldx < d_in ||
      (y_in && ldy < d_out) || n_threads < 1)
    return OR_ERR_ARG;
  for (int i = 0; i < T; ++i) {
    const int a = idx[i];
    if (a < -1 || a >= n_adapters) return OR_ERR_ARG;
    if (a >= 0 && (rank[a] < 0 || (rank[a] > 0 && (!qA[a] || !sA[a] || !qB[a] || !sB[a]))))
      return OR_ERR_ARG;
  }
  if (n_threads > T) n_threads = T > 0 ? T : 1;
  q8_job* jobs = (q8_job*)calloc(n_threads, sizeof(q8_job));
  pthread_t* th = (pthread_t*)calloc(n_threads, sizeof(pthread_t));
  for (int w = 0; w < n_threads; ++w) {
    q8_job j = {dtype, T, d_in, d_out, x, ldx, idx, y_in, ldy, rank, alpha, qA, sA, qB, sB,
                y_out, (int)((long)T * w / n_threads), (int)((long)T * (w + 1) / n_threads)};
    jobs[w] = j;
  }
  for (int w = 1; w < n_threads; ++w) pthread_create(&th[w], NULL, q8_worker, &jobs[w]);
  q8_worker(&jobs[0]);
  for (int w = 1; w < n_threads; ++w) pthread_join(th[w], NULL);
  free(jobs);
  free(th);
  return OR_OK;
}
