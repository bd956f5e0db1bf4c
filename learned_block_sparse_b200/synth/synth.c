/*
 * Seeded synthetic inputs for ETA block-sparse decode (queries, keys, values,
 * predictor weights, per-block offsets, needle positions).
 *
 * This module holds none of the attention method's arithmetic: it only draws
 * numbers and lays them out. Both the CPU oracle (through the tests) and the
 * CUDA path read the bytes it writes, so the two sides always see identical
 * inputs.
 *
 * Generator: Philox4x32-10, the counter-based generator of Salmon, Moraes,
 * Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11).
 * Key = the 64-bit seed; counter = (element-pair index lo, hi, stream id, 0).
 * One Philox call gives four 32-bit words; (w0,w1) and (w2,w3) form two
 * 53-bit uniforms in (0,1), turned into two standard normals by the
 * Box-Muller transform in double precision. Element f of a stream takes
 * normal (f & 1) of call (f >> 1), so any slice can be regenerated on its own.
 *
 * Rounding to storage: double -> fp32 (round to nearest even, the C cast),
 * then fp32 -> bf16 with round to nearest even on the bit pattern.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYN_F32 0
#define SYN_BF16 1

static void philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                          uint32_t k0, uint32_t k1, uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  for (int r = 0; r < 10; ++r) {
    uint64_t p0 = (uint64_t)M0 * c0;
    uint64_t p1 = (uint64_t)M1 * c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += W0; k1 += W1;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* exported for the known-answer test */
void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  philox4x32_10(ctr[0], ctr[1], ctr[2], ctr[3], key[0], key[1], out);
}

static inline double u53(uint32_t lo, uint32_t hi) {
  uint64_t x = ((uint64_t)hi << 32) | lo;
  return ((double)(x >> 11) + 0.5) * (1.0 / 9007199254740992.0); /* in (0,1) */
}

/* standard normal numbers 2*pair (cosine branch) and 2*pair + 1 (sine branch)
 * of stream `stream` under `seed`: one Philox block, Box-Muller in double */
static inline void normal_pair(uint64_t seed, uint32_t stream, uint64_t pair, double* z0, double* z1) {
  uint32_t w[4];
  philox4x32_10((uint32_t)pair, (uint32_t)(pair >> 32), stream, 0u,
                (uint32_t)seed, (uint32_t)(seed >> 32), w);
  double u1 = u53(w[0], w[1]), u2 = u53(w[2], w[3]);
  double r = sqrt(-2.0 * log(u1));
  double th = 6.283185307179586476925286766559 * u2;
  *z0 = r * cos(th);
  *z1 = r * sin(th);
}

/* standard normal number f of stream `stream` under `seed` */
static inline double normal_at(uint64_t seed, uint32_t stream, uint64_t f) {
  double z0, z1;
  normal_pair(seed, stream, f >> 1, &z0, &z1);
  return (f & 1) ? z1 : z0;
}

double synth_normal_at(uint64_t seed, uint32_t stream, uint64_t f) {
  return normal_at(seed, stream, f);
}

static inline uint16_t f32_to_bf16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

static inline void store(void* dst, int dtype, int64_t i, double val) {
  float f = (float)val;
  if (dtype == SYN_F32) ((float*)dst)[i] = f;
  else ((uint16_t*)dst)[i] = f32_to_bf16_rne(f);
}

static inline double load(const void* src, int dtype, int64_t i) {
  if (dtype == SYN_F32) return (double)((const float*)src)[i];
  uint32_t b = (uint32_t)((const uint16_t*)src)[i] << 16;
  float f;
  memcpy(&f, &b, 4);
  return (double)f;
}

/* ---------------------------------------------------------------- threads */

typedef void (*range_fn)(void* ctx, int64_t lo, int64_t hi);
typedef struct { range_fn fn; void* ctx; int64_t lo, hi; } range_job;

static void* run_range(void* p) {
  range_job* j = (range_job*)p;
  j->fn(j->ctx, j->lo, j->hi);
  return NULL;
}

static int g_threads = 0;
void synth_set_threads(int n) { g_threads = n; }

static void parallel_for(int64_t n, range_fn fn, void* ctx) {
  int nt = g_threads > 0 ? g_threads : 1;
  if (nt > 256) nt = 256;
  if (n < 4096 || nt == 1) { fn(ctx, 0, n); return; }
  pthread_t th[256];
  range_job jobs[256];
  for (int t = 0; t < nt; ++t) {
    jobs[t].fn = fn; jobs[t].ctx = ctx;
    jobs[t].lo = n * t / nt; jobs[t].hi = n * (t + 1) / nt;
    if (pthread_create(&th[t], NULL, run_range, &jobs[t]) != 0) { run_range(&jobs[t]); th[t] = 0; }
  }
  for (int t = 0; t < nt; ++t) if (th[t]) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------ plain fills */

typedef struct { uint64_t seed; uint32_t stream; uint64_t f0; double mean, std; int dtype; void* dst; } fill_ctx;

static void fill_range(void* p, int64_t lo, int64_t hi) {
  fill_ctx* c = (fill_ctx*)p;
  for (int64_t i = lo; i < hi; ++i)
    store(c->dst, c->dtype, i, c->mean + c->std * normal_at(c->seed, c->stream, c->f0 + (uint64_t)i));
}

/* dst[i] = mean + std * N_i, i in [0,count), N_i = normal (f0 + i) of the stream */
void synth_normal_fill(uint64_t seed, uint32_t stream, uint64_t f0, int64_t count,
                       double mean, double std, int dtype, void* dst) {
  fill_ctx c = {seed, stream, f0, mean, std, dtype, dst};
  parallel_for(count, fill_range, &c);
}

/* ------------------------------------------------------------- KV caches */

typedef struct {
  uint64_t seed;
  uint32_t stream, off_stream;
  int dtype;
  int64_t B, H, n, cap, d, bs, b0;
  double offset_std;          /* std of the per-block offset vector (0 = none) */
  const void* q;              /* [B][Hq][d] queries in q_dtype, for needles */
  int q_dtype, Hq;
  const int32_t* needles;     /* [B][H][n_needles] block indices, or NULL */
  int n_needles;
  double needle_scale;
  void* dst;                  /* [B][H][cap][d] */
} kv_ctx;

static void kv_range(void* p, int64_t lo, int64_t hi) {
  kv_ctx* c = (kv_ctx*)p;
  const int64_t d = c->d;
  const int G = (int)(c->Hq / c->H);
  double qhat[1024], off[1024], pair_hi = 0.0;
  int64_t cur_bh = -1, cur_off = -1;
  for (int64_t lrow = lo; lrow < hi; ++lrow) {    /* lrow = ((b-b0)*H + h)*n + s */
    const int64_t row = lrow + c->b0 * c->H * c->n;
    int64_t bh = row / c->n, s = row % c->n;
    int64_t b = bh / c->H, h = bh % c->H;
    int64_t blk = s / c->bs;
    int is_needle = 0;
    if (c->needles && c->n_needles > 0) {
      const int32_t* nd = c->needles + bh * c->n_needles;
      for (int j = 0; j < c->n_needles; ++j) if (nd[j] == blk) is_needle = 1;
    }
    if (is_needle && cur_bh != bh) {
      /* unit vector along the first query head of this kv head's group */
      const int64_t qrow = (b * c->Hq + h * G) * d;
      double nrm = 0.0;
      for (int64_t i = 0; i < d; ++i) { double x = load(c->q, c->q_dtype, qrow + i); qhat[i] = x; nrm += x * x; }
      nrm = sqrt(nrm);
      for (int64_t i = 0; i < d; ++i) qhat[i] = nrm > 0.0 ? qhat[i] / nrm : 0.0;
      cur_bh = bh;
    }
    const uint64_t f0 = (uint64_t)row * (uint64_t)d;
    const uint64_t foff = ((uint64_t)bh * (uint64_t)((c->n + c->bs - 1) / c->bs) + (uint64_t)blk) * (uint64_t)d;
    const int64_t o = ((bh - c->b0 * c->H) * c->cap + s) * d;
    if (c->offset_std > 0.0 && (int64_t)foff != cur_off) {
      /* the block's offset vector, drawn once per block */
      for (int64_t i = 0; i < d; ++i) off[i] = normal_at(c->seed, c->off_stream, foff + (uint64_t)i);
      cur_off = (int64_t)foff;
    }
    for (int64_t i = 0; i < d; ++i) {
      double x;
      if ((d & 1) == 0 && (i & 1) == 0) {   /* both numbers of a pair from one draw */
        normal_pair(c->seed, c->stream, (f0 + (uint64_t)i) >> 1, &x, &pair_hi);
      } else if ((d & 1) == 0) {
        x = pair_hi;
      } else {
        x = normal_at(c->seed, c->stream, f0 + (uint64_t)i);
      }
      if (c->offset_std > 0.0) x += c->offset_std * off[i];
      if (is_needle) x += c->needle_scale * qhat[i];
      store(c->dst, c->dtype, o + i, x);
    }
  }
}

/*
 * Fill batches [b0,b1) of a KV cache [B][H][cap][d] for tokens [0,n):
 * standard normal entries, plus an optional per-(b,h,block) offset vector
 * ~ N(0, offset_std^2 I) shared by every key of the block, plus
 * needle_scale * q_hat on every key of the listed needle blocks (q_hat = unit
 * vector of the group's first query head). dst points at batch b0's slice;
 * tokens in [n,cap) are left untouched. q and needles cover all B batches.
 */
void synth_fill_kv(uint64_t seed, uint32_t stream, uint32_t off_stream, int dtype,
                   int64_t B, int64_t H, int64_t n, int64_t cap, int64_t d, int64_t bs,
                   int64_t b0, int64_t b1, double offset_std, const void* q, int q_dtype,
                   int64_t Hq, const int32_t* needles, int n_needles, double needle_scale,
                   void* dst) {
  (void)B;
  kv_ctx c = {seed, stream, off_stream, dtype, B, H, n, cap, d, bs, b0, offset_std,
              q, q_dtype, (int)Hq, needles, n_needles, needle_scale, dst};
  parallel_for((b1 - b0) * H * n, kv_range, &c);
}

/*
 * n_pick distinct block indices in [0, n_range) for each of n_sets sets,
 * drawn from Philox words of the given stream; ascending within a set.
 */
int synth_pick_blocks(uint64_t seed, uint32_t stream, int64_t n_sets, int n_pick,
                      int64_t n_range, int32_t* out) {
  if (n_pick > n_range) return -1;
  for (int64_t s = 0; s < n_sets; ++s) {
    int32_t* o = out + s * n_pick;
    int got = 0;
    for (uint32_t j = 0; got < n_pick; ++j) {
      uint32_t w[4];
      philox4x32_10(j, (uint32_t)s, stream, 1u, (uint32_t)seed, (uint32_t)(seed >> 32), w);
      int32_t cand = (int32_t)(w[0] % (uint32_t)n_range);
      int dup = 0;
      for (int t = 0; t < got; ++t) if (o[t] == cand) dup = 1;
      if (!dup) o[got++] = cand;
    }
    for (int a = 1; a < n_pick; ++a)       /* insertion sort */
      for (int b = a; b > 0 && o[b - 1] > o[b]; --b) { int32_t t = o[b]; o[b] = o[b - 1]; o[b - 1] = t; }
  }
  return 0;
}
