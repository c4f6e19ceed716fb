/*
 * Seeded synthetic inputs: a counter-based SplitMix64 stream turned into
 * standard normals by the Box-Muller transform.
 *
 * This file holds input generation only.  It computes nothing of the
 * attention method; the CUDA path and the CPU oracle both consume the bytes
 * it writes.
 *
 * Definition (so the stream can be re-implemented anywhere):
 *   mix64(z)     : SplitMix64 output function
 *                  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                  z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
 *   GAMMA        : 0x9E3779B97F4A7C15 (SplitMix64 increment)
 *   key          : mix64(seed ^ mix64((stream + 1) * GAMMA))
 *   draw(i)      : mix64(key + (i + 1) * GAMMA), i >= 0; that is the
 *                  (i+1)-th output of SplitMix64 whose state starts at key
 *   normal(e)    : p = e / 2;
 *                  u1 = ((draw(2p) >> 11) + 1) * 2^-53      in (0, 1]
 *                  u2 =  (draw(2p+1) >> 11)      * 2^-53    in [0, 1)
 *                  r  = sqrt(-2 ln u1), t = 2 pi u2   (all in double)
 *                  normal(e) = e even ? r cos t : r sin t
 *   f32 value    : normal(e) rounded to nearest float
 *   bf16 value   : the f32 value rounded to nearest-even bf16
 *   int(i, lo,hi): lo + floor(((draw(i) >> 11) * 2^-53) * (hi - lo + 1))
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define VTGEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed ^ mix64((stream + 1) * VTGEN_GAMMA));
}

static inline uint64_t draw(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * VTGEN_GAMMA);
}

static inline double normal_at(uint64_t key, uint64_t e) {
  const double two_m53 = 1.0 / 9007199254740992.0;
  uint64_t p = e >> 1;
  double u1 = (double)((draw(key, 2 * p) >> 11) + 1) * two_m53;
  double u2 = (double)(draw(key, 2 * p + 1) >> 11) * two_m53;
  double r = sqrt(-2.0 * log(u1));
  double t = 6.283185307179586476925286766559 * u2;
  return (e & 1) ? r * sin(t) : r * cos(t);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  if ((b & 0x7F800000u) == 0x7F800000u) return (uint16_t)(b >> 16); /* inf/nan: not produced */
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

typedef struct {
  uint64_t key;
  int64_t offset;
  int64_t begin, end;
  int kind; /* 0 = f32, 1 = bf16 */
  void* out;
} job_t;

static void* run_job(void* arg) {
  job_t* j = (job_t*)arg;
  for (int64_t i = j->begin; i < j->end; ++i) {
    float f = (float)normal_at(j->key, (uint64_t)(j->offset + i));
    if (j->kind == 0)
      ((float*)j->out)[i] = f;
    else
      ((uint16_t*)j->out)[i] = f32_to_bf16_rne(f);
  }
  return 0;
}

static void run_parallel(uint64_t seed, uint64_t stream, int64_t offset, int64_t count, int kind,
                         void* out, int nthreads) {
  if (count <= 0) return;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (count < 65536) nthreads = 1;
  job_t jobs[256];
  pthread_t th[256];
  uint64_t key = stream_key(seed, stream);
  int64_t chunk = (count + nthreads - 1) / nthreads;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t b = t * chunk, e = b + chunk;
    if (b >= count) break;
    if (e > count) e = count;
    jobs[t].key = key;
    jobs[t].offset = offset;
    jobs[t].begin = b;
    jobs[t].end = e;
    jobs[t].kind = kind;
    jobs[t].out = out;
    if (t == 0 || pthread_create(&th[t], 0, run_job, &jobs[t]) != 0) {
      th[t] = 0;
      if (t != 0) run_job(&jobs[t]);
    }
    started = t + 1;
  }
  run_job(&jobs[0]);
  for (int t = 1; t < started; ++t)
    if (th[t]) pthread_join(th[t], 0);
}

/* Elements [offset, offset+count) of the normal stream (seed, stream) as f32. */
void vtgen_normal_f32(uint64_t seed, uint64_t stream, int64_t offset, int64_t count, float* out,
                      int nthreads) {
  run_parallel(seed, stream, offset, count, 0, out, nthreads);
}

/* Same elements rounded to bf16 (raw uint16 bit patterns). */
void vtgen_normal_bf16(uint64_t seed, uint64_t stream, int64_t offset, int64_t count,
                       uint16_t* out, int nthreads) {
  run_parallel(seed, stream, offset, count, 1, out, nthreads);
}

/* count integers uniform on [lo, hi] inclusive, draws 0..count-1 of (seed, stream). */
void vtgen_uniform_int(uint64_t seed, uint64_t stream, int64_t count, int32_t lo, int32_t hi,
                       int32_t* out) {
  const double two_m53 = 1.0 / 9007199254740992.0;
  uint64_t key = stream_key(seed, stream);
  double span = (double)hi - (double)lo + 1.0;
  for (int64_t i = 0; i < count; ++i) {
    double u = (double)(draw(key, (uint64_t)i) >> 11) * two_m53;
    int64_t v = (int64_t)lo + (int64_t)floor(u * span);
    if (v > hi) v = hi;
    out[i] = (int32_t)v;
  }
}

/* Raw 64-bit draws, exposed so tests can check the stream against its definition. */
void vtgen_raw(uint64_t seed, uint64_t stream, int64_t count, uint64_t* out) {
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < count; ++i) out[i] = draw(key, (uint64_t)i);
}
