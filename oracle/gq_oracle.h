/*
 * gq_oracle.h -- interface of the plain CPU oracle for bucketed gradient quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  The oracle exists to check the CUDA library.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load it; the product path never does.
 * It shares no code, header, table or constant generator with the CUDA library: the config
 * struct below is the oracle's own, with the same meaning as the library's.
 *
 * Sources.  The method comes from three web pages:
 *   [P1] "gradient quantization for communication" (glossary page): the data-parallel step is
 *        Quantize -> Transmit -> Dequantize -> Aggregate, with error feedback.
 *   [P2] "[Paper Review] Optimal Gradient Quantization Condition for Communication-Efficient
 *        Distributed Training": BinGrad-b / BinGrad-pb / ORQ, random rounding, clipping,
 *        buckets of d = 512 (section "Proposed method").
 *   [P3] "Gradient Quantization" (glossary page): max-abs scaling, stochastic rounding and its
 *        0.7 example, QSGD, TernGrad, error feedback.
 * Where the pages leave a step open, the reading used is stated at the function.
 */
#ifndef GQ_ORACLE_H
#define GQ_ORACLE_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_QSGD = 0, OR_TERNGRAD = 1, OR_BINGRAD_B = 2, OR_BINGRAD_PB = 3, OR_ORQ = 4,
       OR_QSGD_NEAREST = 5, /* QSGD levels, deterministic rounding to the nearest level */
       OR_SIGNSGD = 6,      /* scaled sign: levels -m1, +m1, m1 the mean |u| of the bucket */
       OR_QSGD_L2 = 7 };    /* QSGD levels scaled by the bucket's l2 norm instead of max |u| */

typedef struct {
    int32_t scheme;          /* OR_* */
    int32_t levels;          /* s: number of quantization levels */
    int32_t bucket;          /* d: elements per bucket */
    int32_t workers;         /* W */
    int32_t error_feedback;  /* 1: v = g + r and r is updated; 0: v = g */
    float clip_sigma;        /* c > 0: clip to +-c*sigma per bucket; 0: no clipping */
    uint64_t seed;           /* Philox key */
    int64_t n;               /* elements per worker */
} or_config;

/* Philox4x32-10 block function (Salmon, Moraes, Dror, Shaw, SC'11). */
void or_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
/* The uniform in [0,1) drawn for global element index i: the Philox word rounded toward zero to
 * binary32, times 2^-32. */
float or_uniform(uint64_t seed, uint64_t step, uint32_t worker, int64_t i);

/* floor(log2(m)) for finite m > 0, subnormals included. */
int or_fexpo(float m);

/* Per-bucket clipping threshold T = c * sigma (0 if the bucket is all zero). */
float or_clip_threshold(const float *v, int n, float c);
/* Scale m1 of the scaled-sign scheme: the mean of |u| from exact fixed-point sums. */
float or_sign_scale(const float *u, int n);
/* Scale of QSGD-l2: the l2 norm of u from exact fixed-point sums of squares. */
float or_l2_scale(const float *u, int n);

/* 64-point candidate grid and fixed-point positions; returns 0 for a constant bucket. */
int or_grid(const float *u, int n, float grid[64]);

/* Fits, exposed for the oracle's own checks. */
double or_orq_select(const float *u, int n, int s, int *idx_out);
void or_bingrad_b_fit(const float *u, int n, float *a, float *b, float *thr, int *split);
void or_bingrad_pb_fit(const float *u, int n, int *A, int *B, float *ga, float *gb);

/* Bits per code, level-table length and message layout (bytes, codes offset, levels offset). */
int or_bits(int levels);
int or_table_len(int scheme, int levels);
int64_t or_num_buckets(const or_config *cfg);
void or_message_layout(const or_config *cfg, int64_t *bytes, int64_t *codes_off, int64_t *levels_off);

/*
 * One bucket of one worker: fit + round.  v holds the n (<= d) error-fed values of bucket
 * `bucket`.  Outputs: code[n] (level index), q[n] (dequantized value), table[L] (the level
 * table the message carries).  Returns 0 on success.
 */
int or_encode_bucket(const or_config *cfg, int worker, uint64_t step, int64_t bucket,
                     const float *v, int n, uint8_t *code, float *q, float *table);

/* Quantization error over buckets [b0, b1) of one worker: out[0] = sum of the expected
 * squared rounding error, out[1] = sum of u^2, out[2] = realised sum of (Q(u)-u)^2. */
int or_quant_error(const or_config *cfg, int worker, uint64_t step, int64_t b0, int64_t b1,
                   const float *g, const float *r, double *out);

/* Pack n codes of one bucket into d*b/32 words (padding codes are 0). */
void or_pack_bucket(const or_config *cfg, const uint8_t *code, int n, uint32_t *words);
/* Inverse of or_pack_bucket for the first n codes. */
void or_unpack_bucket(const or_config *cfg, const uint32_t *words, int n, uint8_t *code);
/* Base-s packing of the codes: group size g and bits B per group for `levels` (0 if none),
 * code words per bucket, message layout, and the conversions dense <-> base-s message. */
int or_entropy_groups(int levels, int *g, int *B);
int64_t or_entropy_words(const or_config *cfg);
void or_entropy_layout(const or_config *cfg, int64_t *bytes, int64_t *codes_off, int64_t *levels_off);
void or_entropy_pack(const or_config *cfg, const uint8_t *msg, uint8_t *emsg);
void or_entropy_unpack(const or_config *cfg, const uint8_t *emsg, uint8_t *msg);
/* Elias-gamma coding of the codes of odd-s QSGD-family messages (0 if unsupported): layout of
 * the largest message, the conversions (pack returns the bytes used), and one code's length. */
int or_elias_layout(const or_config *cfg, int64_t *cap_bytes, int64_t *offsets_off, int64_t *tables_off,
                    int64_t *stream_off);
int64_t or_elias_pack(const or_config *cfg, const uint8_t *msg, uint8_t *emsg);
int or_elias_unpack(const or_config *cfg, const uint8_t *emsg, uint8_t *msg);
int or_elias_gamma_len(uint32_t x);
/* Dequantize one code with a bucket's level table. */
float or_dequant(const or_config *cfg, const float *table, int code);

/*
 * Whole-vector calls over the bucket range [b0, b1).  Pointers are the full per-worker
 * vectors (indexed by global element index); msg is a full message buffer of
 * or_message_layout bytes.  r may be NULL when error feedback is off.
 */
int or_encode(const or_config *cfg, int worker, uint64_t step, int64_t b0, int64_t b1,
              const float *g, float *r, uint8_t *msg);
int or_decode_accumulate(const or_config *cfg, const uint8_t *const *msgs, int nmsgs,
                         int64_t b0, int64_t b1, float *avg);
int or_fused_step(const or_config *cfg, uint64_t step, int64_t b0, int64_t b1,
                  const float *const *g, float *const *r, uint8_t *const *msgs, float *avg);
/* One bucket of the whole step, from per-bucket slices (see gq_oracle.c). */
int or_fused_bucket(const or_config *cfg, uint64_t step, int64_t bucket, int n,
                    const float *const *g, const float *const *r_in, float *const *r_out,
                    uint32_t *const *words, float *const *tables, float *avg);

/* TernGrad with one scale per parameter tensor (segments [off[t], off[t+1]), off[0] = 0,
 * off[nseg] = n): message layout, encode of one worker (r in/out, NULL without error feedback),
 * decode + average of nmsgs messages. */
void or_tg_layer_layout(const or_config *cfg, int nseg, int64_t *bytes, int64_t *codes_off, int64_t *scales_off);
int or_tg_layer_encode(const or_config *cfg, const int64_t *off, int nseg, int worker, uint64_t step,
                       const float *g, float *r, uint8_t *msg);
int or_tg_layer_decode_accumulate(const or_config *cfg, const int64_t *off, int nseg, const uint8_t *const *msgs,
                                  int nmsgs, float *avg);

#ifdef __cplusplus
}
#endif

#endif
