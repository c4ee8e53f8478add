/*
 * dq_oracle.h -- plain, slow, scalar CPU oracle for the D-Quant hot path.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library. The
 * product library (decode_attention_dq_b200) shares no code, header, table
 * or constant generator with it, and neither includes the other.
 *
 * What it follows:
 *   [news]     "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits"
 *              (English translation of the aimodeling.com news article),
 *              sections "Why Fixed Width Is a Ceiling" and
 *              "Drift: Bending Variable Back to Fixed".
 *   [abstract] "D-Quant: Driftable Entropy Coding for KV Cache Quantization",
 *              Abstract (arXiv 2609.19880).
 * The pages fix: rotation + normalisation make KV coordinates close to
 * N(0,1); symbols are rANS-coded into a fixed-size byte container per token;
 * a stream that is too long is made to fit by "drift" of a few symbols to a
 * cheaper neighbouring level, never more than one level; keys use 8 levels and
 * values 6 at a 2.26-bit budget; the probability model is analytic (no
 * calibration). Every other detail here (level design, rANS parameters,
 * container layout, floating-point order, drift ranking) is a reading of
 * what the pages leave open; each is marked "reading" where it is used.
 *
 * Parity status: every function here is pinned by tests/test_oracle_*.py
 * except dqo_signs' choice of generator use (the pages name no rotation
 * seed): that choice is "parity unpinned" (the splitmix64 generator itself
 * is pinned to its published outputs).
 */
#ifndef DQ_ORACLE_H
#define DQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DQO_D 128            /* head dimension                        */
#define DQO_PROB_BITS 12     /* M = 2^12                              */
#define DQO_M 4096u
#define DQO_L 65536u         /* rANS lower bound, 32-bit state        */
#define DQO_MAX_LEVELS 16
#define DQO_HEADER_BYTES 5   /* fp16 norm + 3-byte final state        */

/* One stream's table (K or V). fp64 design values plus the fp32 values the
 * encoder compares against. */
typedef struct {
  int32_t n_levels;
  int32_t container_bytes;     /* C                                  */
  int32_t payload_bytes;       /* P = C - 2                          */
  int32_t is_lloyd_max;        /* 1: lambda = 0                      */
  double rate;                 /* target bits/value r                */
  double lambda;               /* ECSQ multiplier                    */
  double entropy;              /* H(p) of the design, bits/value     */
  double mse;                  /* E[(u - y_q)^2] for u ~ N(0,1)      */
  double y[DQO_MAX_LEVELS];    /* levels (fp64)                      */
  double t[DQO_MAX_LEVELS];    /* thresholds t_0..t_{n-2} (fp64)     */
  double p[DQO_MAX_LEVELS];    /* cell probabilities                 */
  float yf[DQO_MAX_LEVELS];    /* levels rounded RN to fp32          */
  float tf[DQO_MAX_LEVELS];    /* thresholds rounded RN to fp32      */
  float cost[DQO_MAX_LEVELS];  /* fp32(12 - log2 f_s)                */
  uint32_t freq[DQO_MAX_LEVELS];
  uint32_t cum[DQO_MAX_LEVELS + 1];
} dqo_stream;

typedef struct {
  uint64_t syms_drifted;       /* symbols moved by drift             */
  uint64_t cont_drifted;       /* containers with >= 1 move          */
  uint64_t overflow_fallbacks; /* containers that took the fallback  */
  uint64_t nonfinite_inputs;   /* vectors treated as zero            */
  uint64_t syms_filled;        /* symbols moved up by the RD fill    */
} dqo_stats;

/* ---- tables ---------------------------------------------------------- */
int dqo_lloyd_max(int n, double *y, double *t, double *p, int *iters);
int dqo_ecsq(int n, double lambda, const double *y_init, double *y, double *t,
             double *p, int *iters);
double dqo_entropy(int n, const double *p);
int dqo_int_freqs(int n, const double *p, uint32_t *freq);
int dqo_container_bytes(double bits_per_value);
int dqo_build_stream(int n_levels, int container_bytes, double rate_offset,
                     dqo_stream *out);

/* ---- generator and rotation signs ------------------------------------ */
uint64_t dqo_splitmix64_next(uint64_t *state);
void dqo_signs(uint64_t seed, int head, int8_t *signs /* [128] */);

/* ---- number formats -------------------------------------------------- */
uint16_t dqo_f32_to_f16_rn(float v);
float dqo_f16_to_f32(uint16_t h);
float dqo_bf16_to_f32(uint16_t b);

/* ---- encode steps ---------------------------------------------------- */
void dqo_wht_f32(float *z, int n);
int dqo_rotate_normalize(const float *x, const int8_t *signs, float *u,
                         uint16_t *norm16);
void dqo_quantize(const dqo_stream *st, const float *u, int n, uint8_t *q);
int dqo_rans_encode(const dqo_stream *st, const uint8_t *q, int n,
                    uint8_t *out, int cap);
int dqo_drift_fit(const dqo_stream *st, const float *u, uint8_t *q, int n,
                  int budget, int *moves, uint8_t *moved_mask, int *fallback);
int dqo_encode_vector(const dqo_stream *st, const int8_t *signs,
                      const float *x, uint8_t *container, uint8_t *q_out,
                      dqo_stats *stats);
int dqo_rd_fill(const dqo_stream *st, const float *u, const uint8_t *q0,
                uint8_t *q, int n, int budget, int *ups);
int dqo_encode_vector_mode(const dqo_stream *st, const int8_t *signs,
                           const float *x, uint8_t *container, uint8_t *q_out,
                           dqo_stats *stats, int drift_mode);

/* ---- decode ---------------------------------------------------------- */
int dqo_rans_decode(const dqo_stream *st, const uint8_t *buf, int len,
                    uint8_t *q, int n, uint32_t *x_final, int *consumed);
int dqo_decode_container(const dqo_stream *st, const uint8_t *container,
                         uint8_t *q, uint16_t *norm16);

/* ---- batch helpers (row-major, for the Python side) ------------------ */
int dqo_encode_batch(const dqo_stream *st, const int8_t *signs_per_head,
                     const float *x, const int32_t *head_of, int64_t n_vec,
                     uint8_t *containers, uint8_t *syms, dqo_stats *stats);
int dqo_encode_batch_mode(const dqo_stream *st, const int8_t *signs_per_head,
                          const float *x, const int32_t *head_of, int64_t n_vec,
                          uint8_t *containers, uint8_t *syms, dqo_stats *stats,
                          int drift_mode);
int64_t dqo_decode_batch(const dqo_stream *st, const uint8_t *containers,
                         int64_t n_vec, uint8_t *syms, uint16_t *norm16,
                         int32_t *status);

#ifdef __cplusplus
}
#endif
#endif
