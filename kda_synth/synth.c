/*
 * Seeded synthetic inputs for the KDA + modality-aware short-convolution
 * forward pass.  Shared by the CPU oracle side and the CUDA side; it holds
 * none of the method's arithmetic, only random draws and the value
 * distributions of the workloads:
 *
 *   q, k     ~ N(0,1), then L2-normalised over the head dimension per token
 *   v        ~ N(0,1)
 *   log a    = -softplus(N(0,1)) * scale          (always fp32)
 *   beta     = sigmoid(N(0,1) * beta_std)
 *   weights  ~ N(0, var)                            (fp32)
 *
 * Every element is a pure function of (seed, stream, element index): a
 * counter-based generator (splitmix64 finaliser over a counter, two 53-bit
 * uniforms, Box-Muller cosine branch).  Results therefore do not depend on the
 * thread count, and any slice can be regenerated on its own.
 *
 * bf16 outputs are produced as raw uint16 bit patterns: the double value is
 * rounded to fp32 (round-to-nearest-even) and then to bf16 (RNE).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define SYN_PI 3.14159265358979323846

static inline uint64_t mix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed * 0x100000001B3ull ^ mix64(stream + 0x51ED2701ull));
}

/* standard normal for element `idx` of the stream identified by `key` */
static inline double normal_at(uint64_t key, uint64_t idx) {
  uint64_t h1 = mix64(key ^ mix64(2 * idx));
  uint64_t h2 = mix64(key ^ mix64(2 * idx + 1));
  double u1 = ((double)(h1 >> 11) + 1.0) * (1.0 / 9007199254740992.0); /* (0,1] */
  double u2 = (double)(h2 >> 11) * (1.0 / 9007199254740992.0);         /* [0,1) */
  return sqrt(-2.0 * log(u1)) * cos(2.0 * SYN_PI * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t bias = 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)((u + bias) >> 16);
}

/* dtype codes used by the Python side: 0 = bf16 bits (uint16), 1 = fp32 */
static inline void store(void* out, int dtype, uint64_t i, double x) {
  if (dtype == 0) ((uint16_t*)out)[i] = f32_to_bf16_rne((float)x);
  else ((float*)out)[i] = (float)x;
}

enum { KIND_NORMAL = 0, KIND_NORMAL_ROWNORM = 1, KIND_NEG_SOFTPLUS = 2, KIND_SIGMOID = 3 };

typedef struct {
  int kind;
  uint64_t key;
  uint64_t n_rows;   /* number of rows of `row` elements */
  uint64_t row;      /* row length (head dim for ROWNORM, 1 otherwise) */
  double a, b;       /* kind parameters */
  void* out;
  int dtype;
  uint64_t r0, r1;   /* row range for this worker */
} job_t;

static void* run_job(void* arg) {
  job_t* j = (job_t*)arg;
  double buf[1024];
  for (uint64_t r = j->r0; r < j->r1; ++r) {
    uint64_t base = r * j->row;
    if (j->kind == KIND_NORMAL_ROWNORM) {
      double ss = 0.0;
      for (uint64_t c = 0; c < j->row; ++c) {
        buf[c] = normal_at(j->key, base + c);
        ss += buf[c] * buf[c];
      }
      double inv = 1.0 / sqrt(ss);
      for (uint64_t c = 0; c < j->row; ++c) store(j->out, j->dtype, base + c, buf[c] * inv);
    } else {
      for (uint64_t c = 0; c < j->row; ++c) {
        double z = normal_at(j->key, base + c);
        double x;
        switch (j->kind) {
          case KIND_NORMAL: x = j->a + j->b * z; break;
          case KIND_NEG_SOFTPLUS: {
            /* -softplus(z) * scale, softplus(z) = log(1 + e^z), evaluated stably */
            double sp = z > 0 ? z + log1p(exp(-z)) : log1p(exp(z));
            x = -sp * j->a;
            break;
          }
          default: /* KIND_SIGMOID */
            x = 1.0 / (1.0 + exp(-j->a * z));
            break;
        }
        store(j->out, j->dtype, base + c, x);
      }
    }
  }
  return 0;
}

static int run(int kind, uint64_t seed, uint64_t stream, uint64_t n_rows, uint64_t row,
               double a, double b, void* out, int dtype, int nthreads) {
  if (row == 0 || row > 1024) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((uint64_t)nthreads > n_rows) nthreads = n_rows ? (int)n_rows : 1;
  job_t jobs[256];
  pthread_t th[256];
  uint64_t key = stream_key(seed, stream);
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].kind = kind; jobs[t].key = key; jobs[t].n_rows = n_rows; jobs[t].row = row;
    jobs[t].a = a; jobs[t].b = b; jobs[t].out = out; jobs[t].dtype = dtype;
    jobs[t].r0 = n_rows * (uint64_t)t / (uint64_t)nthreads;
    jobs[t].r1 = n_rows * (uint64_t)(t + 1) / (uint64_t)nthreads;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], 0, run_job, &jobs[t]);
  run_job(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], 0);
  return 0;
}

/* n values ~ N(mean, std^2) */
int syn_normal(uint64_t seed, uint64_t stream, uint64_t n, double mean, double std,
               void* out, int dtype, int nthreads) {
  uint64_t row = 256;
  uint64_t rows = n / row;
  int rc = run(KIND_NORMAL, seed, stream, rows, row, mean, std, out, dtype, nthreads);
  if (rc) return rc;
  /* ragged tail: rows of length 1 starting at rows*row */
  for (uint64_t i = rows * row; i < n; ++i) store(out, dtype, i, mean + std * normal_at(stream_key(seed, stream), i));
  return 0;
}

/* n_rows rows of `row` N(0,1) values, each row scaled to unit L2 norm */
int syn_unit_rows(uint64_t seed, uint64_t stream, uint64_t n_rows, uint64_t row,
                  void* out, int dtype, int nthreads) {
  return run(KIND_NORMAL_ROWNORM, seed, stream, n_rows, row, 0, 0, out, dtype, nthreads);
}

/* n values -softplus(N(0,1)) * scale */
int syn_neg_softplus(uint64_t seed, uint64_t stream, uint64_t n, double scale,
                     void* out, int dtype, int nthreads) {
  uint64_t row = 256;
  uint64_t rows = n / row;
  int rc = run(KIND_NEG_SOFTPLUS, seed, stream, rows, row, scale, 0, out, dtype, nthreads);
  if (rc) return rc;
  uint64_t key = stream_key(seed, stream);
  for (uint64_t i = rows * row; i < n; ++i) {
    double z = normal_at(key, i);
    double sp = z > 0 ? z + log1p(exp(-z)) : log1p(exp(z));
    store(out, dtype, i, -sp * scale);
  }
  return 0;
}

/* n values sigmoid(std * N(0,1)) */
int syn_sigmoid(uint64_t seed, uint64_t stream, uint64_t n, double std,
                void* out, int dtype, int nthreads) {
  uint64_t row = 256;
  uint64_t rows = n / row;
  int rc = run(KIND_SIGMOID, seed, stream, rows, row, std, 0, out, dtype, nthreads);
  if (rc) return rc;
  uint64_t key = stream_key(seed, stream);
  for (uint64_t i = rows * row; i < n; ++i) store(out, dtype, i, 1.0 / (1.0 + exp(-std * normal_at(key, i))));
  return 0;
}
