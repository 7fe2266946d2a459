/*
 * Plain CPU oracle for the hashed N-gram embedding layer ("Over-Encoding").
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call this code:
 * only the tests, the smoke check and the bench's CPU-baseline leg use it.
 * It shares no source with the CUDA library and is deliberately slow and
 * literal: each function writes out one definition from
 * "Scaling Embeddings Outperforms Scaling Experts in Language Models"
 * (LongCat team), section 2 ("N-gram Embedding"), Eq. 2 and Eq. 3.
 *
 * Readings where the paper is silent (shared with the CUDA path as
 * conventions, not as code):
 *   - positions before a sequence start read the pad id 0;
 *   - in Eq. 2 the newest id t_i carries V0^0 (as printed);
 *   - the sum of Eq. 2 is taken as an exact integer before the modulus
 *     (no 64-bit wrap-around);
 *   - H_{n,k} uses the same polynomial for every k, with modulus V_{n,k};
 *   - sub-table order s = (n - 2) * K + (k - 1); W_stacked[o][s*d + c] = W_{n,k}[o][c].
 *
 * Arithmetic: the hash is exact multi-precision integer arithmetic (32-bit
 * limbs), computing the full sum of Eq. 2 and only then reducing it; it does
 * not use Horner's rule. Floating point is fp64 throughout; bf16 and fp32
 * inputs convert to double exactly.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_MAX_N 8
#define ORACLE_LIMBS 8 /* 256 bits: V0 < 2^31 and n <= 8 give X < 2^248 */

/* ---------------- a plain parallel-for over independent items (pthreads) ----------------
 * Items (tokens) are independent; each is computed exactly as in the serial code,
 * so the thread count never changes a result. ORACLE_THREADS overrides the count. */

int oracle_num_threads(void) {
  const char* env = getenv("ORACLE_THREADS");
  if (env && atoi(env) > 0) return atoi(env);
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

typedef void (*item_fn)(int64_t item, void* ctx);
typedef struct {
  item_fn fn;
  void* ctx;
  int64_t n;
  int64_t next; /* next unclaimed item, advanced atomically */
} par_job;

static void* par_worker(void* arg) {
  par_job* job = (par_job*)arg;
  for (;;) {
    const int64_t i = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
    if (i >= job->n) break;
    job->fn(i, job->ctx);
  }
  return NULL;
}

static void par_for(int64_t n, item_fn fn, void* ctx) {
  par_job job = {fn, ctx, n, 0};
  int nt = oracle_num_threads();
  if (nt > 256) nt = 256;
  if (nt > n) nt = (int)(n > 0 ? n : 1);
  pthread_t th[256];
  int started = 0;
  for (int t = 1; t < nt; ++t)
    if (pthread_create(&th[started], NULL, par_worker, &job) == 0) ++started;
  par_worker(&job);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
}

/* ---------------- multi-limb unsigned integers (little-endian 32-bit limbs) ---------------- */

typedef struct { uint32_t w[ORACLE_LIMBS]; } big_t;

static void big_set_small(big_t* a, uint64_t v) {
  memset(a, 0, sizeof(*a));
  a->w[0] = (uint32_t)v;
  a->w[1] = (uint32_t)(v >> 32);
}

/* a = a * m, m < 2^32. Returns nonzero if the product overflowed the limbs. */
static int big_mul_small(big_t* a, uint32_t m) {
  uint64_t carry = 0;
  for (int i = 0; i < ORACLE_LIMBS; ++i) {
    uint64_t p = (uint64_t)a->w[i] * m + carry;
    a->w[i] = (uint32_t)p;
    carry = p >> 32;
  }
  return carry != 0;
}

/* acc = acc + b * m, m < 2^32. Returns nonzero on overflow. */
static int big_add_mul_small(big_t* acc, const big_t* b, uint32_t m) {
  uint64_t carry = 0;
  for (int i = 0; i < ORACLE_LIMBS; ++i) {
    uint64_t p = (uint64_t)b->w[i] * m + (uint64_t)acc->w[i] + carry;
    acc->w[i] = (uint32_t)p;
    carry = p >> 32;
  }
  return carry != 0;
}

/* a mod v (v < 2^31): long division by limbs from the most significant one. */
static uint64_t big_mod_small(const big_t* a, uint64_t v) {
  uint64_t r = 0;
  for (int i = ORACLE_LIMBS - 1; i >= 0; --i) r = ((r << 32) | a->w[i]) % v;
  return r;
}

/*
 * Eq. 2: H_n(t_{i-n+1}, ..., t_i) = (sum_{j=0}^{n-1} t_{i-j} * V0^j) mod V.
 * `window[j]` holds t_{i-j} (j = 0 is the newest id). Returns -1 on bad input.
 */
int64_t oracle_ngram_index(int64_t V0, int n, const int32_t* window, int64_t V) {
  if (n < 1 || n > ORACLE_MAX_N || V0 < 1 || V0 >= ((int64_t)1 << 31) || V < 1 ||
      V >= ((int64_t)1 << 31))
    return -1;
  big_t x, power;
  big_set_small(&x, 0);
  big_set_small(&power, 1); /* V0^0 */
  for (int j = 0; j < n; ++j) {
    if (window[j] < 0) return -1;
    if (big_add_mul_small(&x, &power, (uint32_t)window[j])) return -1; /* x += t_{i-j} * V0^j */
    if (big_mul_small(&power, (uint32_t)V0)) return -1;                  /* power = V0^{j+1} */
  }
  return (int64_t)big_mod_small(&x, (uint64_t)V);
}

/*
 * Context assembly: windows[i*N + j] = t_{i-j} for j = 0..N-1, for every token i.
 * Token i belongs to the sequence b with seq_offsets[b] <= i < seq_offsets[b+1].
 * A position before the start of its sequence reads, if `hist` is given, the
 * sequence's committed history hist[hist_offsets[b] .. hist_offsets[b+1]) from its
 * end backwards, and otherwise (or past the history's start) the pad id 0.
 */
int oracle_context_windows(int N, const int32_t* tokens, const int32_t* seq_offsets,
                           int32_t num_seqs, const int32_t* hist, const int64_t* hist_offsets,
                           int32_t* windows) {
  if (N < 1 || N > ORACLE_MAX_N || num_seqs < 0) return -1;
  for (int32_t b = 0; b < num_seqs; ++b) {
    const int64_t start = seq_offsets[b], end = seq_offsets[b + 1];
    if (end < start) return -1;
    int64_t h_len = 0;
    const int32_t* h = NULL;
    if (hist) {
      h = hist + hist_offsets[b];
      h_len = hist_offsets[b + 1] - hist_offsets[b];
    }
    for (int64_t i = start; i < end; ++i) {
      const int64_t p = i - start; /* position inside the sequence */
      for (int j = 0; j < N; ++j) {
        const int64_t q = p - j;
        int32_t t = 0;
        if (q >= 0)
          t = tokens[start + q];
        else if (h && h_len + q >= 0)
          t = h[h_len + q];
        windows[i * N + j] = t;
      }
    }
  }
  return 0;
}

/*
 * Eq. 2 for every (n, k): idx[i*S + s] = H_{n,k}(window of token i), s = (n-2)*K + (k-1),
 * using the n newest ids of the window and modulus V_nk[s].
 */
int oracle_hash(int64_t V0, int N, int K, const int64_t* V_nk, const int32_t* windows, int64_t T,
                int32_t* idx) {
  if (N < 1 || N > ORACLE_MAX_N || K < 1) return -1;
  const int S = (N - 1) * K;
  int bad = 0;
  for (int64_t i = 0; i < T; ++i) {
    for (int n = 2; n <= N; ++n)
      for (int k = 1; k <= K; ++k) {
        const int s = (n - 2) * K + (k - 1);
        const int64_t r = oracle_ngram_index(V0, n, windows + i * N, V_nk[s]);
        if (r < 0) bad = 1;
        idx[i * S + s] = (int32_t)r;
      }
  }
  return bad ? -1 : 0;
}

static inline double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * Eq. 3 for M tokens given their gathered rows:
 *   out[i][o] = (E0row[i][o] + sum_{s} sum_{c<d} W_stacked[o][s*d + c] * sub[i][s][c]) / (S + 1)
 * with d = D / S. e0rows: [M x D]; subrows: [M x S x d] (row i's sub-rows in order s);
 * W: [D x D] row-major. All in fp64. `is_bf16` selects bf16 (uint16 bits) or fp32 inputs.
 */
typedef struct {
  int is_bf16, D, S, d;
  const void *e0rows, *subrows, *W;
  double* out;
} combine_ctx;

static void combine_one_token(int64_t i, void* p) {
  const combine_ctx* c_ = (const combine_ctx*)p;
  const int is_bf16 = c_->is_bf16, D = c_->D, S = c_->S, d = c_->d;
  const void *e0rows = c_->e0rows, *subrows = c_->subrows, *W = c_->W;
  double* out = c_->out;
  const double inv = 1.0 / (double)(S + 1);
  {
    for (int o = 0; o < D; ++o) {
      double acc = is_bf16 ? bf16_to_double(((const uint16_t*)e0rows)[i * D + o])
                           : (double)((const float*)e0rows)[i * D + o];
      for (int s = 0; s < S; ++s) {
        /* W_{n,k} E_{n,k}(H_{n,k}): the D x d block s of W_stacked times sub-row s. */
        double dot = 0.0;
        for (int c = 0; c < d; ++c) {
          const int64_t wi = (int64_t)o * D + (int64_t)s * d + c;
          const int64_t gi = (i * S + s) * (int64_t)d + c;
          const double w = is_bf16 ? bf16_to_double(((const uint16_t*)W)[wi]) : (double)((const float*)W)[wi];
          const double g = is_bf16 ? bf16_to_double(((const uint16_t*)subrows)[gi])
                                   : (double)((const float*)subrows)[gi];
          dot += w * g;
        }
        acc += dot;
      }
      out[i * D + o] = acc * inv;
    }
  }
}

static int combine(int is_bf16, int D, int S, int64_t M, const void* e0rows, const void* subrows,
                   const void* W, double* out) {
  if (D < 1 || S < 0 || (S > 0 && D % S != 0)) return -1;
  combine_ctx ctx = {is_bf16, D, S, S ? D / S : 0, e0rows, subrows, W, out};
  par_for(M, combine_one_token, &ctx); /* one item per token */
  return 0;
}

int oracle_combine_bf16(int D, int S, int64_t M, const uint16_t* e0rows, const uint16_t* subrows,
                        const uint16_t* W, double* out) {
  return combine(1, D, S, M, e0rows, subrows, W, out);
}

int oracle_combine_f32(int D, int S, int64_t M, const float* e0rows, const float* subrows,
                       const float* W, double* out) {
  return combine(0, D, S, M, e0rows, subrows, W, out);
}

/*
 * The whole layer on host tables: context (pad 0 or history) -> Eq. 2 -> row lookup -> Eq. 3.
 * E_nk: S host pointers, table s of shape [V_nk[s] x d]. E0: [V0 x D]. W: [D x D].
 * elt_bytes: 2 (bf16 bits) or 4 (fp32). out: [T x D] doubles, T = seq_offsets[num_seqs].
 */
int oracle_forward(int elt_bytes, int64_t V0, int D, int N, int K, const int64_t* V_nk,
                   const int32_t* tokens, const int32_t* seq_offsets, int32_t num_seqs,
                   const int32_t* hist, const int64_t* hist_offsets, const void* E0,
                   const void* const* E_nk, const void* W, double* out) {
  if (elt_bytes != 2 && elt_bytes != 4) return -1;
  const int S = (N - 1) * K;
  if (S > 0 && D % S != 0) return -1;
  const int d = S ? D / S : 0;
  const int64_t T = seq_offsets[num_seqs];
  int32_t* windows = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * N + 1));
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * S + 1));
  char* e0rows = (char*)malloc((size_t)elt_bytes * (size_t)(T * D + 1));
  char* subrows = (char*)malloc((size_t)elt_bytes * (size_t)(T * S * d + 1));
  int rc = -1;
  if (!windows || !idx || !e0rows || !subrows) goto done;
  if (oracle_context_windows(N, tokens, seq_offsets, num_seqs, hist, hist_offsets, windows)) goto done;
  if (oracle_hash(V0, N, K, V_nk, windows, T, idx)) goto done;
  for (int64_t i = 0; i < T; ++i) {
    const int32_t t = tokens[i];
    if (t < 0 || t >= V0) goto done;
    memcpy(e0rows + (size_t)elt_bytes * i * D, (const char*)E0 + (size_t)elt_bytes * t * D,
           (size_t)elt_bytes * D);
    for (int s = 0; s < S; ++s)
      memcpy(subrows + (size_t)elt_bytes * ((i * S + s) * d),
             (const char*)E_nk[s] + (size_t)elt_bytes * ((int64_t)idx[i * S + s] * d),
             (size_t)elt_bytes * d);
  }
  rc = combine(elt_bytes == 2, D, S, T, e0rows, subrows, W, out);
done:
  free(windows);
  free(idx);
  free(e0rows);
  free(subrows);
  return rc;
}
