/*
 * infllmv2_oracle.c -- plain, slow CPU oracle for InfLLM v2 block-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the CUDA
 * library is compared against.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark may load it.  It shares no code, header, table or
 * helper with the CUDA path, and the CUDA path never calls it.
 *
 * Sources (all statements below restate them in our own words):
 *  [S]  "MiniCPM4：端设备上的超高效大型语言模型" (MiniCPM4: ultra-efficient LLMs on end
 *       devices, section-by-section summary page):
 *         s2.1.1  the KV cache is cut into block units; every query token picks the
 *                 blocks with the highest relevance score and attends to them only;
 *         s2.1.2  the relevance score between a query token and a KV block is the core;
 *                 each block is represented by fine-grained "semantic kernels"; the
 *                 query heads of one group share one set of top blocks;
 *         s2.1.3  each token computes attention only with the most relevant blocks.
 *  [N]  "OpenBMB publishes Minicpm4: ultra-effective language models for Edge devices
 *       with sparse attention and rapid inference", section "Technical innovations in
 *       MinicPM4": KV blocks, top-k selection through semantic kernels, dynamic
 *       context block selection per token, for prefill and decode.
 *  [W]  The workload definition fixes what the pages leave open: block 64 tokens,
 *       semantic kernel 32 tokens with stride 16, mean-pooled kernels, kernel-to-block
 *       max-pool, group-sum of scores, top-k including 1 initial + 2 local blocks.
 *
 * Readings taken where the pages are silent (R1-R11; each is the plainest reading that
 * the pages and the workload definition support):
 *  R1  a kernel is the arithmetic mean of its key rows; only complete kernels exist;
 *  R2  kernel i covers tokens [i*stride, i*stride + kernel_size);
 *  R3  per head, a softmax over every causally visible kernel; a block's score for the
 *      head is exp(max logit over the block's kernels - lse); the group's score is
 *      the sum over the group's heads;
 *  R4  a block's kernels are all kernels that overlap the block;
 *  R5  kernel i is visible to the query at position t iff its last token is <= t;
 *  R6  forced blocks: the first n_init blocks and the n_local blocks ending at the
 *      query's own block; they count inside top-k;
 *  R7  ties: higher score first, then lower block index;
 *  R8  fewer candidates than slots: take them all and pad with -1;
 *  R9  q-head h belongs to kv-head h / (Hq/Hkv);
 *  R10 default softmax scale 1/sqrt(head_dim) for scoring and attention;
 *  R11 bf16 inputs; kernels stored as bf16 (round to nearest even); scores and
 *      attention in double precision here.
 *
 * Variants of the selection reading (the pages leave the score and the pooling open;
 * [S] s2.1.3 lists hyper-parameter choices without values):
 *  V1  logit-sum scoring: a block's score is the sum over the group's heads of the
 *      block's max scaled logit, with no per-head softmax (one pass, no lse);
 *  V2  inside pooling: a block's kernels are only those lying entirely inside it.
 *  V3  backward: gradients flow to q, k and v through the attention over the selected
 *      blocks; the top-k selection itself passes no gradient.
 *
 * Layouts (row-major, innermost last; bf16 passed as raw uint16 bit patterns):
 *   Q   [B][Lq][Hq][d]      queries are the last Lq tokens of each sequence
 *   K,V [B][Hkv][Lmax][d]
 *   Kc  [B][Hkv][NKmax][d]  NKmax = number of kernels in Lmax tokens
 *   idx [B][Hkv][R][topk]   R = number of evaluated query rows, ascending, -1 padded
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t batch, num_q_heads, num_kv_heads, head_dim;
  int32_t block_size, kernel_size, kernel_stride;
  int32_t topk, n_init, n_local;
  double softmax_scale; /* <= 0 selects 1/sqrt(head_dim) (R10) */
  int32_t score_mode;   /* 0: softmax-sum (R3); 1: logit-sum (V1) */
  int32_t pool_mode;    /* 0: overlapping kernels (R4); 1: kernels inside the block (V2) */
} oracle_params;

/* ---------------------------------------------------------------- bf16 numbers */

static double bf16_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even (R11).  bf16 keeps 8
 * significant bits; its smallest normal is 2^-126 and its subnormal spacing 2^-133. */
static uint16_t bf16_from_double(double x) {
  if (isnan(x)) return 0x7FC0;
  int neg = signbit(x) ? 1 : 0;
  double a = fabs(x);
  uint16_t sign = neg ? 0x8000 : 0;
  if (a == 0.0) return sign;
  if (isinf(a)) return sign | 0x7F80;
  int e;
  frexp(a, &e); /* a = m * 2^e, 0.5 <= m < 1 */
  double quantum = (e - 1 >= -126) ? ldexp(1.0, e - 8) : ldexp(1.0, -133);
  double r = nearbyint(a / quantum) * quantum; /* default rounding mode: nearest even */
  double max_bf16 = ldexp(255.0, 120);         /* (2 - 2^-7) * 2^127 */
  if (r > max_bf16) return sign | 0x7F80;
  float f = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return sign | (uint16_t)(u >> 16);
}

void oracle_bf16_round(const double* x, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_from_double(x[i]);
}

/* ------------------------------------------------------------ sizes and rules */

/* Number of complete kernels in n tokens (R1, R2). */
int64_t oracle_num_kernels(const oracle_params* p, int64_t n) {
  if (n < p->kernel_size) return 0;
  return (n - p->kernel_size) / p->kernel_stride + 1;
}

/* Number of KV blocks holding n tokens ([S] s2.1.1); the last one may be partial. */
int64_t oracle_num_blocks(const oracle_params* p, int64_t n) {
  return (n + p->block_size - 1) / p->block_size;
}

static double scale_of(const oracle_params* p) {
  return p->softmax_scale > 0 ? p->softmax_scale : 1.0 / sqrt((double)p->head_dim);
}

/* R5: kernel i is visible to a query at position t iff its last token is <= t. */
static int kernel_visible(const oracle_params* p, int64_t i, int64_t t) {
  return i * p->kernel_stride + p->kernel_size - 1 <= t;
}

/* Kernel i pools into block j.  R4: their token ranges intersect; V2 (pool_mode 1): the
 * kernel's range lies inside the block's. */
static int kernel_pools_into_block(const oracle_params* p, int64_t i, int64_t j) {
  int64_t k0 = i * p->kernel_stride, k1 = k0 + p->kernel_size; /* [k0, k1) */
  int64_t b0 = j * p->block_size, b1 = b0 + p->block_size;     /* [b0, b1) */
  if (p->pool_mode == 1) return b0 <= k0 && k1 <= b1;
  return k0 < b1 && b0 < k1;
}

/* R6: forced blocks of the query whose own block is cur. */
static int block_forced(const oracle_params* p, int64_t j, int64_t cur) {
  if (j < 0 || j > cur) return 0;
  if (j < p->n_init) return 1;
  if (j > cur - p->n_local) return 1;
  return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------ step 1: compression */

/* Semantic kernels ([S] s2.1.2; R1, R2): Kc[b][g][i] = mean of K rows
 * [i*stride, i*stride + kernel_size), summed exactly in double and rounded once to
 * bf16.  Rows i >= NK(lens[b]) are not written.  lens == NULL means every sequence
 * holds Lmax tokens. */
void oracle_compress(const oracle_params* p, const uint16_t* k, const int32_t* lens,
                     int64_t Lmax, uint16_t* kc) {
  const int64_t B = p->batch, H = p->num_kv_heads, d = p->head_dim;
  const int64_t NKmax = oracle_num_kernels(p, Lmax);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t g = 0; g < H; ++g) {
      int64_t n = lens ? lens[b] : Lmax;
      int64_t nk = oracle_num_kernels(p, n);
      const uint16_t* kbh = k + (b * H + g) * Lmax * d;
      uint16_t* cbh = kc + (b * H + g) * NKmax * d;
      for (int64_t i = 0; i < nk; ++i) {
        for (int64_t c = 0; c < d; ++c) {
          double sum = 0.0;
          for (int64_t r = i * p->kernel_stride; r < i * p->kernel_stride + p->kernel_size; ++r)
            sum += bf16_to_double(kbh[r * d + c]);
          cbh[i * d + c] = bf16_from_double(sum / p->kernel_size);
        }
      }
    }
  }
}

/* ------------------------------------------- steps 2-4: scoring and selection */

typedef struct {
  double score;
  int64_t block;
} candidate;

/* R7: higher score first, then lower block index. */
static int candidate_order(const void* a, const void* b) {
  const candidate* x = (const candidate*)a;
  const candidate* y = (const candidate*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->block > y->block) - (x->block < y->block);
}

/* Block selection for query rows ([S] s2.1.1, s2.1.2; [N]).
 *
 * For every batch b, kv-head g and evaluated row r (query row rows[r] of Q, at
 * position t = n_b - Lq + rows[r]):
 *   x_h(i)  = scale * <q_h, Kc_i>              for each head h of group g, visible i
 *   lse_h   = log sum_i exp(x_h(i))            (R3, R5)
 *   m_h(j)  = max over visible kernels i pooling into block j of x_h(i)  (R4 or V2)
 *   S(j)    = sum over heads h of group g of exp(m_h(j) - lse_h)        (R3, s2.1.2)
 *             or, with logit-sum scoring, of m_h(j)                     (V1)
 * Blocks with no visible pooling kernel are ineligible.  Forced blocks (R6) are taken
 * first; the remaining topk - |forced| slots go to eligible blocks by (R7).  The
 * selection is written ascending and padded with -1 (R8).
 *
 * scores (optional, may be NULL): [B][Hkv][R][nblk_max] doubles, S(j) for eligible
 * blocks, -infinity for ineligible or non-existing ones (a logit-sum may be negative).
 * Returns 0, or -1 when a row's position falls outside its sequence. */
int oracle_select(const oracle_params* p, const uint16_t* q, int64_t Lq, const uint16_t* kc,
                  int64_t NKmax, const int32_t* lens, int64_t Lmax, const int64_t* rows,
                  int64_t n_rows, int32_t* idx, double* scores, int64_t nblk_max) {
  const int64_t B = p->batch, Hq = p->num_q_heads, H = p->num_kv_heads, d = p->head_dim;
  const int64_t G = Hq / H, topk = p->topk;
  const double scale = scale_of(p);
  int bad = 0;
#pragma omp parallel for collapse(3) schedule(dynamic) reduction(| : bad)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t g = 0; g < H; ++g) {
      for (int64_t r = 0; r < n_rows; ++r) {
        int64_t n = lens ? lens[b] : Lmax;
        int64_t t = n - Lq + rows[r];
        int32_t* out = idx + ((b * H + g) * n_rows + r) * topk;
        double* srow = scores ? scores + ((b * H + g) * n_rows + r) * nblk_max : NULL;
        if (srow)
          for (int64_t j = 0; j < nblk_max; ++j) srow[j] = -INFINITY;
        for (int64_t s = 0; s < topk; ++s) out[s] = -1;
        if (t < 0 || t >= n || n > Lmax) {
          bad = 1;
          continue;
        }
        int64_t nk = oracle_num_kernels(p, n);
        int64_t nblk = oracle_num_blocks(p, n);
        int64_t cur = t / p->block_size;

        /* visible kernels and their logits, one head at a time */
        int64_t nvis = 0;
        while (nvis < nk && kernel_visible(p, nvis, t)) ++nvis;
        double* x = (double*)malloc(sizeof(double) * (size_t)(nvis > 0 ? nvis : 1));
        double* S = (double*)calloc((size_t)nblk, sizeof(double));
        char* eligible = (char*)calloc((size_t)nblk, 1);
        for (int64_t hh = 0; hh < G; ++hh) {
          int64_t h = g * G + hh; /* R9 */
          const uint16_t* qv = q + ((b * Lq + rows[r]) * Hq + h) * d;
          double xmax = -INFINITY;
          for (int64_t i = 0; i < nvis; ++i) {
            const uint16_t* kv = kc + ((b * H + g) * NKmax + i) * d;
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += bf16_to_double(qv[c]) * bf16_to_double(kv[c]);
            x[i] = scale * dot;
            if (x[i] > xmax) xmax = x[i];
          }
          if (nvis == 0) continue; /* no kernel is complete yet: nothing to score */
          double lse = 0.0;
          if (p->score_mode == 0) {
            double sum = 0.0;
            for (int64_t i = 0; i < nvis; ++i) sum += exp(x[i] - xmax);
            lse = xmax + log(sum);
          }
          for (int64_t j = 0; j < nblk; ++j) {
            double m = -INFINITY;
            for (int64_t i = 0; i < nvis; ++i)
              if (kernel_pools_into_block(p, i, j) && x[i] > m) m = x[i];
            if (m == -INFINITY) continue;
            eligible[j] = 1;
            S[j] += (p->score_mode == 0) ? exp(m - lse) : m;
          }
        }

        /* forced blocks, then the best eligible remaining ones */
        char* chosen = (char*)calloc((size_t)nblk, 1);
        int64_t n_forced = 0;
        for (int64_t j = 0; j <= cur && j < nblk; ++j)
          if (block_forced(p, j, cur)) {
            chosen[j] = 1;
            ++n_forced;
          }
        candidate* cand = (candidate*)malloc(sizeof(candidate) * (size_t)nblk);
        int64_t nc = 0;
        for (int64_t j = 0; j <= cur && j < nblk; ++j) {
          if (srow && eligible[j]) srow[j] = S[j];
          if (eligible[j] && !chosen[j]) {
            cand[nc].score = S[j];
            cand[nc].block = j;
            ++nc;
          }
        }
        qsort(cand, (size_t)nc, sizeof(candidate), candidate_order);
        int64_t free_slots = topk - n_forced;
        for (int64_t c = 0; c < nc && c < free_slots; ++c) chosen[cand[c].block] = 1;
        int64_t s = 0;
        for (int64_t j = 0; j < nblk && s < topk; ++j)
          if (chosen[j]) out[s++] = (int32_t)j;
        free(cand);
        free(chosen);
        free(eligible);
        free(S);
        free(x);
      }
    }
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------ step 5: sparse attention */

/* Exact attention over the selected blocks ([S] s2.1.3, s2.1.1).
 *
 * For batch b, q-head h (kv-head g = h / G, R9) and evaluated row r at position t:
 *   J = union over the selected blocks j of the keys [j*block, (j+1)*block) with
 *       key position <= t (causal; only the query's own block is cut);
 *   o = sum_{u in J} softmax_u(scale * <q, K_u>) V_u,   lse = log sum_{u in J} exp(...)
 * idx is [B][Hkv][R][topk] for the same rows; -1 entries are ignored and a block
 * listed twice counts once.  o: [B][R][Hq][d] doubles, lse: [B][Hq][R] doubles (may
 * be NULL).  An index outside [0, t / block] is skipped and counted; the count is
 * returned (0 for valid input), or -1 when a row's position is outside its sequence.
 * A row with no key (cannot happen when block 0 is selected) gets o = 0, lse = -inf. */
int64_t oracle_attn(const oracle_params* p, const uint16_t* q, int64_t Lq, const uint16_t* k,
                    const uint16_t* v, const int32_t* lens, int64_t Lmax, const int32_t* idx,
                    const int64_t* rows, int64_t n_rows, double* o, double* lse) {
  const int64_t B = p->batch, Hq = p->num_q_heads, H = p->num_kv_heads, d = p->head_dim;
  const int64_t G = Hq / H, topk = p->topk, bs = p->block_size;
  const double scale = scale_of(p);
  int64_t bad_idx = 0;
  int bad_row = 0;
#pragma omp parallel for collapse(3) schedule(dynamic) reduction(+ : bad_idx) reduction(| : bad_row)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t h = 0; h < Hq; ++h) {
      for (int64_t r = 0; r < n_rows; ++r) {
        int64_t g = h / G;
        int64_t n = lens ? lens[b] : Lmax;
        int64_t t = n - Lq + rows[r];
        double* orow = o + ((b * n_rows + r) * Hq + h) * d;
        for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
        if (lse) lse[(b * Hq + h) * n_rows + r] = -INFINITY;
        if (t < 0 || t >= n || n > Lmax) {
          bad_row = 1;
          continue;
        }
        int64_t cur = t / bs;
        const int32_t* sel = idx + ((b * H + g) * n_rows + r) * topk;
        char* use = (char*)calloc((size_t)(cur + 1), 1);
        for (int64_t s = 0; s < topk; ++s) {
          if (sel[s] < 0) continue;
          if (sel[s] > cur) {
            ++bad_idx;
            continue;
          }
          use[sel[s]] = 1;
        }
        /* gather the keys of the selected blocks, in position order */
        int64_t nkeys = 0;
        for (int64_t j = 0; j <= cur; ++j)
          if (use[j]) nkeys += (j == cur) ? (t - j * bs + 1) : bs;
        int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nkeys > 0 ? nkeys : 1));
        double* logit = (double*)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
        int64_t u = 0;
        for (int64_t j = 0; j <= cur; ++j)
          if (use[j])
            for (int64_t key = j * bs; key < (j + 1) * bs && key <= t; ++key) pos[u++] = key;
        const uint16_t* qv = q + ((b * Lq + rows[r]) * Hq + h) * d;
        const uint16_t* kbase = k + (b * H + g) * Lmax * d;
        const uint16_t* vbase = v + (b * H + g) * Lmax * d;
        double mx = -INFINITY;
        for (u = 0; u < nkeys; ++u) {
          double dot = 0.0;
          for (int64_t c = 0; c < d; ++c)
            dot += bf16_to_double(qv[c]) * bf16_to_double(kbase[pos[u] * d + c]);
          logit[u] = scale * dot;
          if (logit[u] > mx) mx = logit[u];
        }
        if (nkeys > 0) {
          double den = 0.0;
          for (u = 0; u < nkeys; ++u) den += exp(logit[u] - mx);
          for (u = 0; u < nkeys; ++u) {
            double w = exp(logit[u] - mx) / den;
            for (int64_t c = 0; c < d; ++c) orow[c] += w * bf16_to_double(vbase[pos[u] * d + c]);
          }
          if (lse) lse[(b * Hq + h) * n_rows + r] = mx + log(den);
        }
        free(logit);
        free(pos);
        free(use);
      }
    }
  }
  if (bad_row) return -1;
  return bad_idx;
}

/* --------------------------------------- step 6: backward of the sparse attention */

/* Gradients of the sparse attention of oracle_attn with respect to q, k and v, for a
 * given upstream gradient d_o ([S] s2.1 and s2.1.3: the attention is trained, so it is
 * differentiated; the block selection is a top-k choice, constant almost everywhere, so
 * no gradient flows through it -- the block lists are fixed inputs here (V3)).
 *
 * For batch b, q-head h (kv-head g = h / G) and query row r at position t, with J the
 * keys of the selected blocks cut at t and P_u = softmax_u(scale * <q, K_u>) over J:
 *   dV_u  += P_u d_o                          (u in J)
 *   dP_u   = <d_o, V_u>
 *   dS_u   = P_u (dP_u - sum_w P_w dP_w)
 *   dq     = scale * sum_u dS_u K_u
 *   dK_u  += scale * dS_u q
 * Every query row of the Lq rows is evaluated (queries are the last Lq tokens of each
 * sequence, as in oracle_attn); idx is [B][Hkv][Lq][topk].
 *   d_o [B][Lq][Hq][d] bf16; dq [B][Lq][Hq][d] doubles; dk, dv [B][Hkv][Lmax][d]
 *   doubles (rows a sequence does not reach stay 0).
 *   o   [B][Lq][Hq][d] doubles or NULL: the forward output, when the backward takes it as
 *       an input; then sum_w P_w dP_w is computed as <d_o, o> (equal for the exact o).
 * Returns 0, the count of block indices outside [0, t / block] (skipped), or -1 when a
 * row's position lies outside its sequence.  Parallel over (b, kv-head) only, so the
 * sums into dk and dv run in a fixed order. */
int64_t oracle_attn_backward(const oracle_params* p, const uint16_t* q, int64_t Lq, const uint16_t* k,
                             const uint16_t* v, const int32_t* lens, int64_t Lmax, const int32_t* idx,
                             const uint16_t* d_o, const double* o, double* dq, double* dk, double* dv) {
  const int64_t B = p->batch, Hq = p->num_q_heads, H = p->num_kv_heads, d = p->head_dim;
  const int64_t G = Hq / H, topk = p->topk, bs = p->block_size;
  const double scale = scale_of(p);
  int64_t bad_idx = 0;
  int bad_row = 0;
  memset(dq, 0, sizeof(double) * (size_t)(B * Lq * Hq * d));
  memset(dk, 0, sizeof(double) * (size_t)(B * H * Lmax * d));
  memset(dv, 0, sizeof(double) * (size_t)(B * H * Lmax * d));
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(+ : bad_idx) reduction(| : bad_row)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t g = 0; g < H; ++g) {
      int64_t n = lens ? lens[b] : Lmax;
      const uint16_t* kbase = k + (b * H + g) * Lmax * d;
      const uint16_t* vbase = v + (b * H + g) * Lmax * d;
      double* dkb = dk + (b * H + g) * Lmax * d;
      double* dvb = dv + (b * H + g) * Lmax * d;
      for (int64_t r = 0; r < Lq; ++r) {
        int64_t t = n - Lq + r;
        if (t < 0 || t >= n || n > Lmax) {
          bad_row = 1;
          continue;
        }
        int64_t cur = t / bs;
        const int32_t* sel = idx + ((b * H + g) * Lq + r) * topk;
        char* use = (char*)calloc((size_t)(cur + 1), 1);
        for (int64_t s = 0; s < topk; ++s) {
          if (sel[s] < 0) continue;
          if (sel[s] > cur) {
            ++bad_idx;
            continue;
          }
          use[sel[s]] = 1;
        }
        int64_t nkeys = 0;
        for (int64_t j = 0; j <= cur; ++j)
          if (use[j]) nkeys += (j == cur) ? (t - j * bs + 1) : bs;
        int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nkeys > 0 ? nkeys : 1));
        double* pr = (double*)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
        double* dp = (double*)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
        int64_t u = 0;
        for (int64_t j = 0; j <= cur; ++j)
          if (use[j])
            for (int64_t key = j * bs; key < (j + 1) * bs && key <= t; ++key) pos[u++] = key;
        for (int64_t hh = 0; hh < G && nkeys > 0; ++hh) {
          int64_t h = g * G + hh; /* R9 */
          const uint16_t* qv = q + ((b * Lq + r) * Hq + h) * d;
          const uint16_t* gv = d_o + ((b * Lq + r) * Hq + h) * d;
          double* dqv = dq + ((b * Lq + r) * Hq + h) * d;
          /* probabilities */
          double mx = -INFINITY;
          for (u = 0; u < nkeys; ++u) {
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += bf16_to_double(qv[c]) * bf16_to_double(kbase[pos[u] * d + c]);
            pr[u] = scale * dot;
            if (pr[u] > mx) mx = pr[u];
          }
          double den = 0.0;
          for (u = 0; u < nkeys; ++u) den += exp(pr[u] - mx);
          for (u = 0; u < nkeys; ++u) pr[u] = exp(pr[u] - mx) / den;
          /* dP_u = <d_o, V_u>, and the row's sum_u P_u dP_u */
          double pdp = 0.0;
          for (u = 0; u < nkeys; ++u) {
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += bf16_to_double(gv[c]) * bf16_to_double(vbase[pos[u] * d + c]);
            dp[u] = dot;
            pdp += pr[u] * dot;
          }
          if (o) { /* the forward output as given: sum_w P_w dP_w = <d_o, o> */
            const double* ov = o + ((b * Lq + r) * Hq + h) * d;
            pdp = 0.0;
            for (int64_t c = 0; c < d; ++c) pdp += bf16_to_double(gv[c]) * ov[c];
          }
          for (u = 0; u < nkeys; ++u) {
            const double ds = pr[u] * (dp[u] - pdp);
            for (int64_t c = 0; c < d; ++c) {
              dqv[c] += scale * ds * bf16_to_double(kbase[pos[u] * d + c]);
              dkb[pos[u] * d + c] += scale * ds * bf16_to_double(qv[c]);
              dvb[pos[u] * d + c] += pr[u] * bf16_to_double(gv[c]);
            }
          }
        }
        free(dp);
        free(pr);
        free(pos);
        free(use);
      }
    }
  }
  if (bad_row) return -1;
  return bad_idx;
}
