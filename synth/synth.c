/*
 * Seeded synthetic attention inputs for video-diffusion self-attention.
 *
 * This is test and benchmark infrastructure shared by the CPU oracle and the
 * GPU path. It holds none of the attention method's arithmetic: it only draws
 * the Q, K, V tensors, in the packed [total_tokens, H, D] layout with bf16
 * elements stored as uint16 bit patterns.
 *
 * Recipe (one reading of the diffusion workloads the skip-softmax pages
 * describe: WAN 2.2 video latents on a T x Hh x Ww token grid):
 *   - tokens of sequence b are row-major over its (t, y, x) grid, x fastest,
 *     and sit at packed rows cu[b] .. cu[b+1]-1;
 *   - Q = N(0,1) + amp * PE and K = N(0,1) + amp * PE (independent noise per
 *     tensor, token, head and dim), V = N(0,1);
 *   - PE is one 3-D sinusoidal code shared by all heads: D splits into
 *     [t | y | x] with d_y = d_x = 2*floor(D/6) and d_t = D - 2*d_y; on an
 *     axis with d_a dims and position p, dim 2i is sin(p * 10000^(-2i/d_a))
 *     and dim 2i+1 is cos of the same angle;
 *   - normals come from a counter-based splitmix64 stream (Steele, Lea and
 *     Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014)
 *     turned into pairs by the Box-Muller transform; element e of a tensor
 *     takes member (e & 1) of pair e >> 1, so every element is a pure
 *     function of (seed, tensor, e) and any slice can be drawn alone;
 *   - each value is computed in double, rounded to float, then to bf16 with
 *     round-to-nearest-even.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* i-th output of the splitmix64 stream whose state starts at `key`. */
uint64_t synth_splitmix64(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * GOLDEN_GAMMA);
}

static inline uint64_t tensor_key(uint64_t seed, int tensor) {
  return mix64(seed * GOLDEN_GAMMA + 0x632BE59BD9B4E019ULL * (uint64_t)(tensor + 1));
}

/* Standard normal for element e of the tensor stream `key`. */
static inline double normal_at(uint64_t key, uint64_t e) {
  const uint64_t pair = e >> 1;
  const uint64_t a = synth_splitmix64(key, 2 * pair);
  const uint64_t b = synth_splitmix64(key, 2 * pair + 1);
  const double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53; /* (0, 1] */
  const double u2 = (double)(b >> 11) * 0x1.0p-53;         /* [0, 1) */
  const double r = sqrt(-2.0 * log(u1));
  const double ang = 6.283185307179586476925286766559 * u2;
  return (e & 1) ? r * sin(ang) : r * cos(ang);
}

uint16_t synth_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

double synth_normal(uint64_t seed, int tensor, uint64_t e) { return normal_at(tensor_key(seed, tensor), e); }

/* Positional code value of dim d for grid position (t, y, x). */
double synth_pe(int D, int t, int y, int x, int d) {
  const int dyx = 2 * (D / 6);
  const int dt = D - 2 * dyx;
  int p, da, i2;
  if (d < dt) { p = t; da = dt; i2 = d; }
  else if (d < dt + dyx) { p = y; da = dyx; i2 = d - dt; }
  else { p = x; da = dyx; i2 = d - dt - dyx; }
  const int i = i2 / 2;
  const double ang = (double)p * pow(10000.0, -2.0 * (double)i / (double)da);
  return (i2 & 1) ? cos(ang) : sin(ang);
}

typedef struct {
  uint64_t seed;
  double amp;
  int H, D, nseq;
  const int32_t* grids;
  const int64_t* starts;
  uint16_t *q, *k, *v;
  int64_t tok_begin, tok_end;
} job_t;

static void* run_job(void* arg) {
  const job_t* j = (const job_t*)arg;
  const uint64_t kq = tensor_key(j->seed, 0), kk = tensor_key(j->seed, 1), kv = tensor_key(j->seed, 2);
  double* pe = (double*)malloc(sizeof(double) * (size_t)j->D);
  int b = 0;
  for (int64_t n = j->tok_begin; n < j->tok_end; ++n) {
    while (b + 1 < j->nseq && n >= j->starts[b + 1]) ++b;
    const int64_t local = n - j->starts[b];
    const int Hh = j->grids[3 * b + 1], Ww = j->grids[3 * b + 2];
    const int x = (int)(local % Ww);
    const int y = (int)((local / Ww) % Hh);
    const int t = (int)(local / ((int64_t)Ww * Hh));
    for (int d = 0; d < j->D; ++d) pe[d] = synth_pe(j->D, t, y, x, d);
    for (int h = 0; h < j->H; ++h) {
      const uint64_t base = ((uint64_t)n * (uint64_t)j->H + (uint64_t)h) * (uint64_t)j->D;
      for (int d = 0; d < j->D; ++d) {
        const uint64_t e = base + (uint64_t)d;
        if (j->q) j->q[e] = synth_bf16_rne((float)(normal_at(kq, e) + j->amp * pe[d]));
        if (j->k) j->k[e] = synth_bf16_rne((float)(normal_at(kk, e) + j->amp * pe[d]));
        if (j->v) j->v[e] = synth_bf16_rne((float)normal_at(kv, e));
      }
    }
  }
  free(pe);
  return NULL;
}

/*
 * Fill q, k, v (each [total_tokens, H, D] uint16 bf16 patterns; any may be
 * NULL to skip it). grids holds nseq triples (T, Hh, Ww); total_tokens is
 * the sum of their products. Returns the number of tokens written, or -1.
 */
int64_t synth_qkv(uint64_t seed, double amp, int H, int D, int nseq, const int32_t* grids,
                  uint16_t* q, uint16_t* k, uint16_t* v, int nthreads) {
  if (H <= 0 || D <= 0 || (D & 1) || nseq <= 0 || !grids) return -1;
  int64_t* starts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nseq + 1));
  starts[0] = 0;
  for (int b = 0; b < nseq; ++b) {
    const int64_t s = (int64_t)grids[3 * b] * grids[3 * b + 1] * grids[3 * b + 2];
    if (s < 0) { free(starts); return -1; }
    starts[b + 1] = starts[b] + s;
  }
  const int64_t total = starts[nseq];
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  job_t jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = (job_t){seed, amp, H, D, nseq, grids, starts, q, k, v,
                      total * i / nthreads, total * (i + 1) / nthreads};
    pthread_create(&th[i], NULL, run_job, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(starts);
  return total;
}
