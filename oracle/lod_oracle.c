/*
 * lod_oracle.c -- plain, slow CPU oracle for Level-of-Detail (LoD) attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant table with
 * the CUDA library: it is written from the method's description alone.
 *
 * Source of every step: "Level of Detail Attention: allocating resolution
 * instead of sparsity" (featherless.ai blog), section "How It Works":
 *   - paragraph 1: after every chunk of 256 tokens the keys are grouped into
 *     centroid clusters; each cluster is cut into pages of 16 keys; the cache
 *     is then a three-tier view (group averages, page averages, raw keys).
 *   - paragraph 2: a query scores itself against the centroids, opens the top
 *     eight groups, scores the page summaries of those groups, opens the top
 *     two pages of each, and attends exactly to their keys, to the most recent
 *     block sliding window of 256-512 tokens and to one or more sink tokens.
 *   - paragraph 3: exact pairs and a coarse remainder share ONE softmax; an
 *     unopened group enters as its average key and value repeated by its key
 *     count, and the unopened pages of opened groups enter the same way.
 *   - paragraph 4: with zero-variance groups this equals full attention, and
 *     otherwise the coarse terms never overstate a group's attention mass.
 *
 * Where the page is silent the oracle takes these readings (each one is also
 * listed with its reason in the design notes of the repository):
 *   R-kmeans  plain k-means (squared Euclidean distance) on the cached keys;
 *             seeded farthest-first initialisation: the first centre is the key
 *             at local index splitmix64(seed ^ ((unit << 32) + chunk)) mod n,
 *             every later centre is the key whose distance to the nearest
 *             chosen centre is largest (ties: lower local index); then
 *             `iters` Lloyd rounds of (assign, ties -> lower cluster id;
 *             centre := mean of its members, an empty cluster keeps its
 *             centre).  The final groups are the last assignment and their
 *             summaries are exact member means.
 *   R-sinks   sink positions [0, S) are never clustered; chunk 0 clusters the
 *             remaining chunk - S keys, so every position is counted once.
 *   R-pages   a group's members in ascending position, cut into runs of
 *             `page` keys (the last run may be short); page slots are numbered
 *             group-major within a chunk.
 *   R-store   summaries are sums in high precision, divided by the count and
 *             rounded (round-to-nearest-even) to the cache dtype.
 *   R-window  the window is block granular: a query at t with block bt =
 *             t / chunk sees exactly [chunk * max(0, bt - W/chunk + 1), t];
 *             the sinks are [0, min(S, window start)); the index visible to it
 *             is the complete chunks before the window start.
 *   R-rank    groups are ranked by scale * q.k_mean (no count term), ties to
 *             the lower global group id (chunk * k + slot); pages by
 *             scale * q.k_page_mean, ties to the lower page slot; a group with
 *             no more pages than `top_pages` is opened entirely.
 *   R-twotier top_pages = 0 is the pages' two-tier LoD ("Level of Detail
 *             Attention", the quality tables' "Two-tier LoD" rows): an opened
 *             group is opened whole, with no page tier and no page remainder.
 *   R-coarse  every unopened page of an opened group is its own coarse entry
 *             (mean key logit + ln(count), mean value); ln(count) is added
 *             after the 1/sqrt(d) scale, since n copies of exp(x) are
 *             exp(x + ln n).
 *   R-int4    three-tier INT4 ("Level of Detail Attention", the paragraph
 *             after the quality tables: the centroids keep similar keys
 *             together, so the cache can be stored at INT4, and in the
 *             three-tier mode only the selected pages are decompressed): the
 *             member keys and values of every page are stored as 4-bit codes
 *             of a per-page, per-channel asymmetric quantiser.  For page p and
 *             channel j over the page's members: low = min x, scale =
 *             (max x - low) / 15 in fp32, code = clamp(rint((x - low) /
 *             scale), 0, 15) (0 when scale = 0), and the decompressed value is
 *             fmaf(code, scale, low) in fp32.  Opened pages' exact entries use
 *             the decompressed keys and values; the summaries, the sinks and
 *             the window keep the cache values.
 *   R-prec    decisions that turn floating point into an integer (the k-means
 *             argmin and argmax, the top-k rankings) are taken in fp32, the
 *             precision of the GPU kernels; every softmax, mean and output is
 *             computed in fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL -1
#define ORC_ENOMEM -2

typedef struct {
  int32_t d;          /* head dimension */
  int32_t chunk;      /* tokens per indexed chunk (256 on the page) */
  int32_t page;       /* keys per page (16 on the page) */
  int32_t clusters;   /* k: groups per chunk */
  int32_t iters;      /* Lloyd rounds */
  int32_t top_groups; /* groups opened per query (8 on the page) */
  int32_t top_pages;  /* pages opened per opened group (2 on the page); 0:
                         every page (two-tier LoD, opened groups go whole) */
  int32_t window;     /* sliding window in tokens, a multiple of chunk */
  int32_t sinks;      /* number of sink tokens at the start */
  int32_t store_bf16; /* 1: summaries rounded to bfloat16, 0: to float32 */
  uint64_t seed;      /* k-means initialisation seed */
  double scale;       /* softmax scale applied to q.k; <= 0 means 1/sqrt(d) */
} orc_params;

/* Page slots reserved per chunk: chunk/page full pages plus one short page per
 * group at most, so chunk/page + k always suffices. */
int32_t orc_page_slots(const orc_params* p) { return p->chunk / p->page + p->clusters; }

/* SplitMix64 output for a generator state x (Steele, Lea, Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014): advance the state
 * by the golden-ratio increment, then apply the variant-13 finaliser. */
uint64_t orc_splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Round a real number to the nearest bfloat16 (8 significant bits), ties to
 * even, returned as a double.  Written from the definition of the format:
 * for |x| in [2^(e-1), 2^e) the spacing of representable values is 2^(e-8).
 * (Normal range only; the summaries never approach the subnormal range.) */
double orc_round_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  frexp(x, &e); /* |x| = m * 2^e with m in [0.5, 1) */
  double ulp = ldexp(1.0, e - 8);
  double r = nearbyint(x / ulp) * ulp; /* default mode: ties to even */
  return r;
}

static double round_store(const orc_params* p, double x) {
  return p->store_bf16 ? orc_round_bf16(x) : (double)(float)x;
}

static double scale_of(const orc_params* p) {
  return p->scale > 0.0 ? p->scale : 1.0 / sqrt((double)p->d);
}

/* Squared Euclidean distance in fp32 (the decision precision). */
static float dist2_f32(const float* a, const float* b, int d) {
  float s = 0.0f;
  for (int i = 0; i < d; ++i) {
    float t = a[i] - b[i];
    s += t * t;
  }
  return s;
}

static double dist2_f64(const float* a, const float* b, int d) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) {
    double t = (double)a[i] - (double)b[i];
    s += t * t;
  }
  return s;
}

static double rel_margin(double best, double second) {
  double den = best > 1e-30 ? best : 1e-30;
  return (second - best) / den;
}

/*
 * Build the index of ONE sequence (one batch entry, one KV head): chunks
 * [0, nchunks) of keys K[T][d] and values V[T][d] (float, already holding the
 * cache-dtype values).  unit = b * Hkv + kvh enters the initialisation seed.
 *
 * Outputs (caller-allocated; P = orc_page_slots):
 *   assign    [nchunks*chunk]   group slot of each position, -1 for sinks
 *   gK, gV    [nchunks*k*d]     group mean key / value (rounded), 0 if empty
 *   gCnt      [nchunks*k]       group sizes
 *   pK, pV    [nchunks*P*d]     page mean key / value (rounded), 0 if unused
 *   pCnt      [nchunks*P]       page sizes (0 = unused slot)
 *   pBeg      [nchunks*P]       first member of the page, offset into perm
 *   gPage     [nchunks*(k+1)]   pages of group j are slots [gPage[j], gPage[j+1])
 *   perm      [nchunks*chunk]   chunk-local positions, group-major, ascending
 *                               within a group; -1 past the clustered keys
 *   init_idx  [nchunks*k]       local indices chosen by the initialisation
 *   min_margin[nchunks]         smallest relative margin of any k-means
 *                               decision in the chunk (fragility measure)
 *   key_margin[nchunks*chunk]   relative margin (second - best) / best of each
 *                               key's last assignment; +inf for sinks
 *   objective [nchunks*iters]   sum of squared distances after each
 *                               assignment step (nullable)
 */
int orc_build_sequence(const orc_params* p, uint64_t unit, const float* K, const float* V,
                       int64_t nchunks, int32_t* assign, double* gK, double* gV, int32_t* gCnt,
                       double* pK, double* pV, int32_t* pCnt, int32_t* pBeg, int32_t* gPage,
                       int32_t* perm, int32_t* init_idx, double* min_margin, double* key_margin,
                       double* objective) {
  const int d = p->d, C = p->chunk, k = p->clusters, P = orc_page_slots(p);
  if (d <= 0 || C <= 0 || k <= 0 || p->page <= 0 || p->sinks < 0 || p->sinks >= C || p->iters < 1)
    return ORC_EINVAL;
  float* cen = (float*)malloc(sizeof(float) * (size_t)k * d);
  float* mind = (float*)malloc(sizeof(float) * (size_t)C);
  int32_t* a = (int32_t*)malloc(sizeof(int32_t) * (size_t)C);
  double* acc = (double*)malloc(sizeof(double) * (size_t)d);
  double* accv = (double*)malloc(sizeof(double) * (size_t)d);
  int32_t* cnt = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
  if (!cen || !mind || !a || !acc || !accv || !cnt) {
    free(cen); free(mind); free(a); free(acc); free(accv); free(cnt);
    return ORC_ENOMEM;
  }

  for (int64_t c = 0; c < nchunks; ++c) {
    const int first = (c == 0) ? p->sinks : 0; /* R-sinks */
    const int n = C - first;
    const float* xs = K + ((size_t)c * C + first) * d;
    const float* vs = V + ((size_t)c * C + first) * d;
    double margin = INFINITY;

    for (int i = 0; i < C; ++i) {
      assign[c * C + i] = -1;
      key_margin[c * C + i] = INFINITY;
    }

    /* --- seeded farthest-first initialisation (R-kmeans) --- */
    for (int i = 0; i < n; ++i) mind[i] = INFINITY;
    for (int j = 0; j < k; ++j) {
      int pick;
      if (j == 0) {
        uint64_t h = orc_splitmix64(p->seed ^ ((unit << 32) + (uint64_t)c));
        pick = (int)(h % (uint64_t)n);
      } else {
        pick = 0;
        for (int i = 1; i < n; ++i)
          if (mind[i] > mind[pick]) pick = i; /* strict: ties keep the lower index */
        /* fragility: the winner against the best strictly smaller value */
        float second = -INFINITY;
        for (int i = 0; i < n; ++i)
          if (mind[i] < mind[pick] && mind[i] > second) second = mind[i];
        if (second > -INFINITY) {
          /* larger is better here, so the margin is taken relative to the winner */
          double m = ((double)mind[pick] - (double)second) /
                     ((double)mind[pick] > 1e-30 ? (double)mind[pick] : 1e-30);
          if (m < margin) margin = m;
        }
      }
      init_idx[c * k + j] = pick;
      memcpy(cen + (size_t)j * d, xs + (size_t)pick * d, sizeof(float) * d);
      for (int i = 0; i < n; ++i) {
        float dd = dist2_f32(xs + (size_t)i * d, cen + (size_t)j * d, d);
        if (dd < mind[i]) mind[i] = dd;
      }
    }

    /* --- Lloyd rounds: assign, then move each centre to its members' mean --- */
    for (int it = 0; it < p->iters; ++it) {
      double obj = 0.0;
      for (int i = 0; i < n; ++i) {
        int bj = 0;
        float bd = dist2_f32(xs + (size_t)i * d, cen, d);
        float sd = INFINITY;
        for (int j = 1; j < k; ++j) {
          float dd = dist2_f32(xs + (size_t)i * d, cen + (size_t)j * d, d);
          if (dd < bd) { sd = bd; bd = dd; bj = j; }
          else if (dd < sd) sd = dd;
        }
        a[i] = bj;
        if (k > 1) {
          double m = rel_margin((double)bd, (double)sd);
          if (m < margin) margin = m;
          key_margin[c * C + first + i] = m;
        }
        obj += dist2_f64(xs + (size_t)i * d, cen + (size_t)bj * d, d);
      }
      if (objective) objective[c * p->iters + it] = obj;
      for (int j = 0; j < k; ++j) {
        int m = 0;
        for (int t = 0; t < d; ++t) acc[t] = 0.0;
        for (int i = 0; i < n; ++i)
          if (a[i] == j) {
            ++m;
            for (int t = 0; t < d; ++t) acc[t] += (double)xs[(size_t)i * d + t];
          }
        if (m > 0)
          for (int t = 0; t < d; ++t) cen[(size_t)j * d + t] = (float)(acc[t] / m);
      }
    }
    min_margin[c] = margin;

    /* --- groups, pages and their summaries (R-pages, R-store) --- */
    int slot = 0, off = 0;
    for (int j = 0; j < k; ++j) {
      cnt[j] = 0;
      for (int i = 0; i < n; ++i)
        if (a[i] == j) cnt[j]++;
    }
    for (int i = 0; i < C; ++i) perm[c * C + i] = -1;
    for (int q = 0; q < P; ++q) {
      pCnt[c * P + q] = 0;
      pBeg[c * P + q] = 0;
      for (int t = 0; t < d; ++t) pK[((size_t)c * P + q) * d + t] = pV[((size_t)c * P + q) * d + t] = 0.0;
    }
    for (int j = 0; j < k; ++j) {
      gPage[c * (k + 1) + j] = slot;
      gCnt[c * k + j] = cnt[j];
      for (int t = 0; t < d; ++t) acc[t] = accv[t] = 0.0;
      int inpage = 0, pstart = off;
      for (int i = 0; i < n; ++i) {
        if (a[i] != j) continue;
        assign[c * C + first + i] = j;
        perm[c * C + off] = first + i;
        ++off;
        ++inpage;
        if (inpage == p->page) { /* close a full page */
          pBeg[c * P + slot] = pstart;
          pCnt[c * P + slot] = inpage;
          ++slot;
          pstart = off;
          inpage = 0;
        }
      }
      if (inpage > 0) {
        pBeg[c * P + slot] = pstart;
        pCnt[c * P + slot] = inpage;
        ++slot;
      }
      /* group means */
      for (int i = 0; i < n; ++i)
        if (a[i] == j)
          for (int t = 0; t < d; ++t) {
            acc[t] += (double)xs[(size_t)i * d + t];
            accv[t] += (double)vs[(size_t)i * d + t];
          }
      for (int t = 0; t < d; ++t) {
        gK[((size_t)c * k + j) * d + t] = cnt[j] ? round_store(p, acc[t] / cnt[j]) : 0.0;
        gV[((size_t)c * k + j) * d + t] = cnt[j] ? round_store(p, accv[t] / cnt[j]) : 0.0;
      }
    }
    gPage[c * (k + 1) + k] = slot;
    /* page means, from the member lists just written */
    for (int q = 0; q < slot; ++q) {
      int b0 = pBeg[c * P + q], m = pCnt[c * P + q];
      for (int t = 0; t < d; ++t) acc[t] = accv[t] = 0.0;
      for (int r = 0; r < m; ++r) {
        int loc = perm[c * C + b0 + r];
        for (int t = 0; t < d; ++t) {
          acc[t] += (double)K[((size_t)c * C + loc) * d + t];
          accv[t] += (double)V[((size_t)c * C + loc) * d + t];
        }
      }
      for (int t = 0; t < d; ++t) {
        pK[((size_t)c * P + q) * d + t] = round_store(p, acc[t] / m);
        pV[((size_t)c * P + q) * d + t] = round_store(p, accv[t] / m);
      }
    }
  }
  free(cen); free(mind); free(a); free(acc); free(accv); free(cnt);
  return ORC_OK;
}

/*
 * Page quantiser of R-int4 for one sequence.  X: [nchunks*chunk][d] cache
 * values (keys or values); pCnt/pBeg/perm: the index of orc_build_sequence.
 * Outputs, member-ordered like perm (row m of chunk c is the token at offset
 * perm[c*chunk + m]):
 *   code  [nchunks*chunk][d]  one 4-bit code per byte (0 past the members)
 *   scale [nchunks*P][d]      per page slot and channel (0 for unused slots)
 *   low   [nchunks*P][d]
 */
int orc_quantize_pages(const orc_params* p, const float* X, int64_t nchunks, const int32_t* pCnt,
                       const int32_t* pBeg, const int32_t* perm, uint8_t* code, float* scale,
                       float* low) {
  const int d = p->d, C = p->chunk, P = orc_page_slots(p);
  if (d <= 0 || C <= 0) return ORC_EINVAL;
  memset(code, 0, (size_t)nchunks * C * d);
  for (int64_t c = 0; c < nchunks; ++c)
    for (int q = 0; q < P; ++q) {
      const int64_t pid = c * P + q;
      const int m = pCnt[pid], b0 = pBeg[pid];
      for (int j = 0; j < d; ++j) {
        scale[pid * d + j] = 0.0f;
        low[pid * d + j] = 0.0f;
      }
      if (m <= 0) continue;
      if (b0 < 0 || b0 + m > C) return ORC_EINVAL;
      for (int j = 0; j < d; ++j) {
        float lo = INFINITY, hi = -INFINITY;
        for (int r = 0; r < m; ++r) {
          const float x = X[(c * C + perm[c * C + b0 + r]) * (int64_t)d + j];
          if (x < lo) lo = x;
          if (x > hi) hi = x;
        }
        const float sc = (hi - lo) / 15.0f;
        scale[pid * d + j] = sc;
        low[pid * d + j] = lo;
        for (int r = 0; r < m; ++r) {
          const float x = X[(c * C + perm[c * C + b0 + r]) * (int64_t)d + j];
          float v = sc > 0.0f ? rintf((x - lo) / sc) : 0.0f;
          if (v < 0.0f) v = 0.0f;
          if (v > 15.0f) v = 15.0f;
          code[(c * C + b0 + r) * (int64_t)d + j] = (uint8_t)v;
        }
      }
    }
  return ORC_OK;
}

/* Per-row bookkeeping returned by orc_attend_row, for the invariant tests. */
typedef struct {
  int64_t n_exact;         /* exact (position) entries */
  int64_t n_coarse_groups; /* coarse entries standing for unopened groups */
  int64_t n_coarse_pages;  /* coarse entries standing for unopened pages */
  int64_t covered;         /* positions accounted for, counts included */
  int64_t n_visible;       /* visible non-empty groups */
  double weight_sum;       /* sum of the normalised softmax weights */
  double window_start;     /* first window position */
} orc_row_stats;

typedef struct {
  double s64;   /* scale * q.k in fp64 (softmax logit before ln count) */
  float s32;    /* the same score in fp32 (the ranking decision) */
  int64_t id;   /* global id used for tie breaks */
  int32_t pos;  /* owner data: chunk or slot */
} ranked;

static double dot64(const float* q, const double* k, int d) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) s += (double)q[i] * k[i];
  return s;
}
static float dot32(const float* q, const double* k, int d) {
  float s = 0.0f;
  for (int i = 0; i < d; ++i) s += q[i] * (float)k[i];
  return s;
}
static double dot64f(const float* q, const float* k, int d) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) s += (double)q[i] * (double)k[i];
  return s;
}

/* Better = larger fp32 score, then lower id (R-rank). */
static int better(const ranked* x, const ranked* y) {
  if (x->s32 != y->s32) return x->s32 > y->s32;
  return x->id < y->id;
}

/* Plain selection sort of the first m entries (m is small: top-k). */
static void take_top(ranked* r, int n, int m) {
  for (int i = 0; i < m && i < n; ++i) {
    int b = i;
    for (int j = i + 1; j < n; ++j)
      if (better(&r[j], &r[b])) b = j;
    ranked t = r[i]; r[i] = r[b]; r[b] = t;
  }
}

/*
 * LoD attention for ONE query row at position t.  K, V: [>t][d] float (cache
 * values); the index arrays are those produced by orc_build_sequence (or an
 * index imported from elsewhere, in the same layout) for chunks
 * [0, nchunks_built).  forced_groups [top_groups] / forced_pages
 * [top_groups*top_pages] (nullable, -1 padded) replace the rankings when
 * given.  Outputs: out[d] (fp64), lse, sel_groups[top_groups] (global group
 * ids c*k+j, best first, -1 padded), sel_pages[top_groups*top_pages]
 * (chunk-global page slots c*P+slot), stats.
 */
int orc_attend_row_q(const orc_params* p, const float* q, int64_t t, const float* K, const float* V,
                     int64_t nchunks_built, const double* gK, const double* gV, const int32_t* gCnt,
                     const double* pK, const double* pV, const int32_t* pCnt, const int32_t* pBeg,
                     const int32_t* gPage, const int32_t* perm, const uint8_t* kcode,
                     const float* kscale, const float* klow, const uint8_t* vcode,
                     const float* vscale, const float* vlow, const int32_t* forced_groups,
                     const int32_t* forced_pages, double* out, double* lse, int32_t* sel_groups,
                     int32_t* sel_pages, orc_row_stats* st) {
  const int d = p->d, C = p->chunk, k = p->clusters, P = orc_page_slots(p);
  const int G = p->top_groups, TP = p->top_pages;
  const double sc = scale_of(p);
  const float sc32 = (float)sc;
  if (t < 0 || p->window <= 0 || p->window % C || G < 1 || G > 64 || TP < 0 || TP > 64)
    return ORC_EINVAL;

  /* R-window */
  const int64_t bt = t / C, nw = p->window / C;
  const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;
  const int64_t ws = wb * C;
  const int64_t nvis = wb; /* chunks [0, wb) are visible through the index */
  const int64_t ns = p->sinks < ws ? p->sinks : ws;
  if (nvis > nchunks_built) return ORC_EINVAL;

  /* all entries of the single softmax: logit, value pointer (f or d), multiplicity */
  int64_t cap = (t + 1) + nvis * k + (int64_t)G * P + 8;
  double* lg = (double*)malloc(sizeof(double) * cap);
  const float** vf = (const float**)malloc(sizeof(float*) * cap);
  const double** vd = (const double**)malloc(sizeof(double*) * cap);
  int64_t* mult = (int64_t*)malloc(sizeof(int64_t) * cap);
  ranked* gr = (ranked*)malloc(sizeof(ranked) * (nvis * k + 1));
  ranked* pr = (ranked*)malloc(sizeof(ranked) * (P + 1));
  char* opened = (char*)calloc((size_t)(nvis * k + 1), 1);
  /* R-int4: decompressed member rows of the opened pages (keys, then values) */
  const int quant = kcode && kscale && klow && vcode && vscale && vlow;
  float* deq = quant ? (float*)malloc(sizeof(float) * 2 * (size_t)(G * C + 1) * d) : NULL;
  if (!lg || !vf || !vd || !mult || !gr || !pr || !opened || (quant && !deq)) {
    free(lg); free(vf); free(vd); free(mult); free(gr); free(pr); free(opened); free(deq);
    return ORC_ENOMEM;
  }
  int64_t ndeq = 0;
  int64_t ne = 0;
  orc_row_stats s = {0};
  s.window_start = (double)ws;

  /* exact: sinks and the window */
  for (int64_t i = 0; i < ns; ++i) {
    lg[ne] = sc * dot64f(q, K + i * d, d); vf[ne] = V + i * d; vd[ne] = 0; mult[ne] = 1; ++ne;
  }
  for (int64_t i = ws; i <= t; ++i) {
    lg[ne] = sc * dot64f(q, K + i * d, d); vf[ne] = V + i * d; vd[ne] = 0; mult[ne] = 1; ++ne;
  }
  s.n_exact = ne;

  /* group scores over the visible, non-empty groups */
  int ng = 0;
  for (int64_t c = 0; c < nvis; ++c)
    for (int j = 0; j < k; ++j) {
      int64_t id = c * k + j;
      if (gCnt[id] <= 0) continue;
      gr[ng].s64 = sc * dot64(q, gK + id * d, d);
      gr[ng].s32 = dot32(q, gK + id * d, d) * sc32;
      gr[ng].id = id;
      gr[ng].pos = (int32_t)c;
      ++ng;
    }
  s.n_visible = ng;

  /* choose the opened groups */
  int nopen = 0;
  int64_t open_ids[64];
  if (forced_groups) {
    for (int i = 0; i < G; ++i)
      if (forced_groups[i] >= 0) open_ids[nopen++] = forced_groups[i];
  } else {
    take_top(gr, ng, G);
    nopen = ng < G ? ng : G;
    for (int i = 0; i < nopen; ++i) open_ids[i] = gr[i].id;
  }
  for (int i = 0; i < G; ++i) sel_groups[i] = i < nopen ? (int32_t)open_ids[i] : -1;
  for (int i = 0; i < G * TP; ++i) sel_pages[i] = -1;
  for (int i = 0; i < nopen; ++i) opened[open_ids[i]] = 1;

  /* coarse: unopened groups */
  for (int i = 0; i < ng; ++i) {
    int64_t id = gr[i].id;
    if (opened[id]) continue;
    lg[ne] = gr[i].s64 + log((double)gCnt[id]);
    vf[ne] = 0; vd[ne] = gV + id * d; mult[ne] = gCnt[id]; ++ne;
    s.n_coarse_groups++;
  }

  /* opened groups: page scores, top pages exact, the rest coarse */
  for (int i = 0; i < nopen; ++i) {
    int64_t id = open_ids[i];
    int64_t c = id / k;
    int j = (int)(id % k);
    int p0 = gPage[c * (k + 1) + j], p1 = gPage[c * (k + 1) + j + 1];
    int np = 0;
    for (int sl = p0; sl < p1; ++sl) {
      int64_t pid = c * P + sl;
      pr[np].s64 = sc * dot64(q, pK + pid * d, d);
      pr[np].s32 = dot32(q, pK + pid * d, d) * sc32;
      pr[np].id = sl;
      pr[np].pos = sl;
      ++np;
    }
    int nopen_p = 0;
    int32_t op[64];
    if (TP == 0) {  /* two-tier LoD: an opened group is opened whole */
      for (int r = 0; r < np; ++r) op[nopen_p++] = pr[r].pos;
    } else if (forced_pages) {
      for (int r = 0; r < TP; ++r) {
        int32_t f = forced_pages[i * TP + r];
        if (f >= 0) op[nopen_p++] = (int32_t)(f - c * P);
      }
    } else {
      take_top(pr, np, TP);
      nopen_p = np < TP ? np : TP;
      for (int r = 0; r < nopen_p; ++r) op[r] = pr[r].pos;
    }
    for (int r = 0; r < nopen_p && r < TP; ++r) sel_pages[i * TP + r] = (int32_t)(c * P + op[r]);
    for (int r = 0; r < np; ++r) {
      int sl = pr[r].pos, is_open = 0;
      for (int u = 0; u < nopen_p; ++u) is_open |= (op[u] == sl);
      int64_t pid = c * P + sl;
      if (is_open) {
        for (int m = 0; m < pCnt[pid]; ++m) {
          int64_t pos = c * C + perm[c * C + pBeg[pid] + m];
          if (quant) {
            float* kh = deq + (size_t)(2 * ndeq) * d;
            float* vh = kh + d;
            const int64_t row = (c * C + pBeg[pid] + m) * (int64_t)d;
            for (int j = 0; j < d; ++j) {
              kh[j] = fmaf((float)kcode[row + j], kscale[pid * d + j], klow[pid * d + j]);
              vh[j] = fmaf((float)vcode[row + j], vscale[pid * d + j], vlow[pid * d + j]);
            }
            ++ndeq;
            lg[ne] = sc * dot64f(q, kh, d); vf[ne] = vh; vd[ne] = 0; mult[ne] = 1; ++ne;
          } else {
            lg[ne] = sc * dot64f(q, K + pos * d, d); vf[ne] = V + pos * d; vd[ne] = 0; mult[ne] = 1; ++ne;
          }
          s.n_exact++;
        }
      } else {
        lg[ne] = pr[r].s64 + log((double)pCnt[pid]);
        vf[ne] = 0; vd[ne] = pV + pid * d; mult[ne] = pCnt[pid]; ++ne;
        s.n_coarse_pages++;
      }
    }
  }

  /* the single softmax (fp64) */
  double m = -INFINITY;
  for (int64_t e = 0; e < ne; ++e) if (lg[e] > m) m = lg[e];
  double L = 0.0;
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int64_t e = 0; e < ne; ++e) {
    double w = exp(lg[e] - m);
    L += w;
    for (int i = 0; i < d; ++i) out[i] += w * (vf[e] ? (double)vf[e][i] : vd[e][i]);
    s.covered += mult[e];
  }
  for (int i = 0; i < d; ++i) out[i] /= L;
  *lse = m + log(L);
  double ws_ = 0.0;
  for (int64_t e = 0; e < ne; ++e) ws_ += exp(lg[e] - m) / L;
  s.weight_sum = ws_;
  if (st) *st = s;
  free(lg); free(vf); free(vd); free(mult); free(gr); free(pr); free(opened); free(deq);
  return ORC_OK;
}

/* orc_attend_row_q with the opened pages read in the cache values. */
int orc_attend_row(const orc_params* p, const float* q, int64_t t, const float* K, const float* V,
                   int64_t nchunks_built, const double* gK, const double* gV, const int32_t* gCnt,
                   const double* pK, const double* pV, const int32_t* pCnt, const int32_t* pBeg,
                   const int32_t* gPage, const int32_t* perm, const int32_t* forced_groups,
                   const int32_t* forced_pages, double* out, double* lse, int32_t* sel_groups,
                   int32_t* sel_pages, orc_row_stats* st) {
  return orc_attend_row_q(p, q, t, K, V, nchunks_built, gK, gV, gCnt, pK, pV, pCnt, pBeg, gPage, perm,
                          NULL, NULL, NULL, NULL, NULL, NULL, forced_groups, forced_pages, out, lse,
                          sel_groups, sel_pages, st);
}

/* Full softmax attention of one query at position t over keys [0, t], fp64. */
int orc_dense_row(const orc_params* p, const float* q, int64_t t, const float* K, const float* V,
                  double* out, double* lse) {
  const int d = p->d;
  const double sc = scale_of(p);
  double m = -INFINITY;
  for (int64_t i = 0; i <= t; ++i) {
    double l = sc * dot64f(q, K + i * d, d);
    if (l > m) m = l;
  }
  double L = 0.0;
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int64_t i = 0; i <= t; ++i) {
    double w = exp(sc * dot64f(q, K + i * d, d) - m);
    L += w;
    for (int j = 0; j < d; ++j) out[j] += w * (double)V[i * d + j];
  }
  for (int j = 0; j < d; ++j) out[j] /= L;
  *lse = m + log(L);
  return ORC_OK;
}

/* Element-wise orc_round_bf16 over an array (test helper). */
void orc_round_bf16_array(const double* in, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_round_bf16(in[i]);
}
