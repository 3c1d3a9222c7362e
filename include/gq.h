/*
 * gq.h -- C ABI of the B200 library for bucketed gradient quantization (libgq.so).
 *
 * The library implements the data-parallel step that the page "gradient quantization for
 * communication" (glossary) describes in its section "How Gradient Quantization Works":
 * Quantize -> Transmit -> Dequantize -> Aggregate, with the error feedback of its section
 * "Quantization Schemes".  Quantize is bucketed (buckets of d elements, the review
 * "[Paper Review] Optimal Gradient Quantization Condition for Communication-Efficient
 * Distributed Training", section "Proposed method") with one of five level fits:
 *   QSGD-s and TernGrad (max-abs scaling; "Gradient Quantization" glossary),
 *   BinGrad-b, BinGrad-pb and ORQ-s (the review's proposed schemes).
 * W workers are W separate buffers on one GPU; "Transmit" is the message each worker writes to
 * device memory, and Dequantize + Aggregate read it back (or, in gq_fused_step, never leave
 * the chip).
 *
 * Conventions for every call:
 *   - Pointers named "device" are CUDA device (or managed) memory owned by the caller, 16-byte
 *     aligned.  Arrays of pointers (grads[], residuals[], msgs[]) are HOST arrays of W device
 *     pointers.  The library keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only enqueue
 *     work; results are ready when the stream is.  Calls on one plan must not overlap on the
 *     GPU (the plan's status word is shared).
 *   - Argument errors are reported synchronously (GQ_ERR_INVALID / GQ_ERR_UNSUPPORTED) and
 *     nothing is enqueued.  A launch failure returns GQ_ERR_CUDA.  Non-finite input does not
 *     fail the call: it raises a flag on the plan that gq_plan_status reports; the outputs of
 *     the affected bucket are then unspecified (but every access stays in bounds).
 *   - The library never allocates inside a call except gq_plan_create.
 *   - With n = 0 every call is a no-op that returns GQ_OK; data pointers may then be NULL.
 */
#ifndef GQ_H
#define GQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GQ_API __attribute__((visibility("default")))
#else
#define GQ_API
#endif

#define GQ_MAX_WORKERS 64
#define GQ_MIN_BUCKET 128
#define GQ_MAX_BUCKET 32768
#define GQ_MAX_LEVELS 16
/* Largest level count of the QSGD family (QSGD, QSGD-nearest, QSGD-l2): 129 .. 256 levels take
 * 8-bit codes (255 levels with nearest rounding is symmetric INT8). */
#define GQ_MAX_QSGD_LEVELS 256

typedef enum {
    GQ_QSGD = 0,       /* s uniform levels on [-m, m], m = max|u| of the bucket, stochastic rounding */
    GQ_TERNGRAD = 1,   /* QSGD with s = 3: levels {-m, 0, m} */
    GQ_BINGRAD_B = 2,  /* two levels at the side means of the SSE-optimal split, deterministic */
    GQ_BINGRAD_PB = 3, /* two grid levels at least as far apart as BinGrad-b's, minimising the expected squared
                        * error among such pairs; stochastic inside, clamped outside */
    GQ_ORQ = 4,        /* s levels: {min, max} plus s-2 greedy picks from a 64-point grid, stochastic rounding */
    /* Biased baselines ("Gradient Quantization" glossary, "Deterministic vs stochastic rounding"
     * and "Ternary and binary quantization"); buckets of d <= 512 only: */
    GQ_QSGD_NEAREST = 5, /* the QSGD-s levels and message, each value rounded to its nearest level (ties to the
                          * upper one), no randomness; s = 3 is deterministic TernGrad, s = 15 symmetric INT4 */
    GQ_SIGNSGD = 6,      /* scaled sign: levels -m1 and +m1, m1 = mean |u| of the bucket (exact fixed-point
                          * sum), code 1 for u >= 0; 1 bit per element */
    /* QSGD as published (l2 scaling; the glossary's QSGD, whose codes are Elias-coded), d <= 512: */
    GQ_QSGD_L2 = 7,      /* the QSGD-s levels and stochastic rounding with m = ||u||_2 of the bucket (exact
                          * fixed-point sum of squares) in place of max |u|; sparse codes for gq_elias_pack */
    /* TernGrad with one scale per parameter tensor (the glossary's "single scaling factor per
     * layer"); needs the tensors' offsets (gq_plan_set_segments); no clipping: */
    GQ_TERNGRAD_LAYER = 8
} gq_scheme_t;

typedef enum {
    GQ_OK = 0,
    GQ_ERR_INVALID = 1,     /* an argument is out of range, NULL where required, or misaligned */
    GQ_ERR_UNSUPPORTED = 2, /* a valid combination this build does not implement */
    GQ_ERR_CUDA = 3,        /* a CUDA call failed (launch, allocation of the plan's status word) */
    GQ_ERR_NONFINITE = 4,   /* gq_plan_status: some input value was NaN or infinite */
    GQ_ERR_NOMEM = 5,       /* host allocation failed */
    GQ_ERR_TIMEOUT = 6      /* gq_plan_status: a kernel's bounded wait for a bulk copy gave up */
} gq_status_t;

/*
 * Configuration of a plan.
 *   scheme         gq_scheme_t.
 *   levels         s.  QSGD: 2..16.  TernGrad: 3 (0 means 3).  BinGrad-b/pb: 2 (0 means 2).
 *                  ORQ: 2..16.  QSGD-nearest, QSGD-l2: 2..16.  SignSGD: 2 (0 means 2).  Codes take
 *                  b = ceil(log2 s) bits (1..4).
 *   bucket         d, elements per bucket: a power of two in [128, 32768] (at most 512 for
 *                  QSGD-nearest, SignSGD and QSGD-l2: GQ_ERR_UNSUPPORTED above).  The vector is cut
 *                  into ceil(n/d) buckets; the last one may hold fewer than d elements.
 *   workers        W in [1, 64] for gq_fused_step (gq_encode ignores it).
 *   error_feedback 1: v = g + r is quantized and r <- v - Q(v); 0: v = g, no residual.
 *   clip_sigma     c >= 0.  c > 0 clips each bucket to [-c*sigma, c*sigma] before the fit
 *                  (sigma: the bucket's population standard deviation); the residual keeps the
 *                  clipped part.  0 disables clipping.
 *   seed           key of the Philox4x32-10 stream used for stochastic rounding.
 *   n              elements per worker, 0 <= n < 2^40.
 */
typedef struct {
    int32_t scheme;
    int32_t levels;
    int32_t bucket;
    int32_t workers;
    int32_t error_feedback;
    float clip_sigma;
    uint64_t seed;
    int64_t n;
} gq_config_t;

typedef struct gq_plan *gq_plan_t; /* opaque; owned by the library */

/* Validate a configuration without touching any device.  GQ_OK if a plan can be made. */
GQ_API gq_status_t gq_config_check(const gq_config_t *cfg);

/*
 * Layout of one worker's message, the bytes a worker would transmit (host computation, no
 * device needed).  *bytes: total size.  *codes_off: offset of the packed codes, ceil(n/d)
 * buckets of d*b/32 uint32 words each.  *levels_off: offset (16-byte aligned) of the level
 * tables, ceil(n/d) tables of L float32 each (L = 1 for the QSGD family: the scale m;
 * 2 for BinGrad-b/pb and SignSGD: the two levels; s for ORQ: the ascending levels).
 * Packing inside a bucket: dense, in element order, least significant bit first: bit j of the
 * code (the index of its level) of element e is bit (b*e + j) % 32 of word (b*e + j) / 32 of
 * the bucket's words.  Padding elements of the last bucket have code 0.
 * Any output pointer may be NULL.
 */
GQ_API gq_status_t gq_message_layout(const gq_config_t *cfg, size_t *bytes, size_t *codes_off, size_t *levels_off);

/* Create a plan: validates cfg, selects kernels and allocates on the current device the plan's
 * 4-byte status word and the scratch of gq_quant_error (the only device allocations the library
 * makes).  The plan must be used on that device only. */
GQ_API gq_status_t gq_plan_create(const gq_config_t *cfg, gq_plan_t *out);
/* Free the plan (synchronous; the caller must make sure no work of the plan is pending). */
GQ_API gq_status_t gq_plan_destroy(gq_plan_t plan);

/*
 * Quantize: one worker's gradient into its message (the "Quantize" step, with error feedback).
 *   worker    Philox worker index of this gradient (any 32-bit value; the draws for element i
 *             are keyed on (seed, step, worker, i)).
 *   step      training step; its low 32 bits key the draws.
 *   grad      device, n float32, read only.
 *   residual  device, n float32, read and overwritten with v - Q(v); must be NULL iff the
 *             plan's error_feedback is 0.
 *   msg       device, gq_message_layout bytes, written completely.
 */
GQ_API gq_status_t gq_encode(gq_plan_t plan, uint32_t worker, uint64_t step, const float *grad, float *residual,
                      void *msg, void *stream);

/*
 * Dequantize + Aggregate: avg[i] = (sum over w = 0..nmsgs-1, in that order, of the level of
 * element i in msgs[w]) * (1/nmsgs), in float32.
 *   msgs      host array of nmsgs (1..64) device pointers to messages written by gq_encode
 *             or gq_fused_step with this plan's configuration.
 *   avg       device, n float32, overwritten.
 */
GQ_API gq_status_t gq_decode_accumulate(gq_plan_t plan, const void *const *msgs, int nmsgs, float *avg, void *stream);

/*
 * The whole step for the plan's W workers: worker w (w = 0..W-1, Philox worker index w) is
 * quantized as by gq_encode and the mean of the W dequantized gradients is written to avg,
 * as by gq_decode_accumulate; the dequantized values never leave the chip (for d <= 512 they
 * are summed in registers; for larger buckets one CTA walks a bucket's W workers and keeps the
 * running sum in shared memory, or, above d = 8192, in avg's own slice while it stays in L2).
 *   grads      host array of W device pointers (n float32 each).
 *   residuals  host array of W device pointers (in/out), or NULL iff error_feedback is 0.
 *   msgs       host array of W device pointers receiving the messages, or NULL not to write
 *              messages.
 *   avg        device, n float32, overwritten.
 */
GQ_API gq_status_t gq_fused_step(gq_plan_t plan, uint64_t step, const float *const *grads, float *const *residuals,
                          void *const *msgs, float *avg, void *stream);

/*
 * Quantization error of one worker's gradient, for measuring how much a fit loses (the
 * expected quantization variance the review's ORQ minimises, section "Proposed method").  The
 * fit and the rounding are those of gq_encode (same worker, step and draws); nothing but `out`
 * is written and the residual is only read.
 *   out   device, 3 doubles: out[0] = sum over elements of the expected squared rounding error
 *         p (b - u)^2 + (1 - p) (a - u)^2 given the fitted levels (u the value quantized after
 *         clipping, [a, b] its bracket, p its probability of rounding up; (b - u)(u - a) for
 *         unbiased rounding), out[1] = sum of u^2, out[2] = sum of (Q(u) - u)^2 for this
 *         step's draws.  Binary64; each bucket's sums are reduced in a fixed order, so the
 *         result does not depend on the launch shape.
 * Uses the plan's error scratch of 24 * (ceil(n/d) + ceil(ceil(n/d) / 4096)) bytes.
 */
GQ_API gq_status_t gq_quant_error(gq_plan_t plan, uint32_t worker, uint64_t step, const float *grad,
                                  const float *residual, double *out, void *stream);

/*
 * Allocation-free variant of gq_quant_error.  There is no counterpart in the paper: this entry
 * point exists for callers that cannot call cudaMalloc -- code running inside a framework's
 * caching allocator or memory pool (which must not be re-entered), processes whose device
 * memory is reserved up front, plugins that are handed buffers but no allocator.  Such callers
 * cannot create a plan (gq_plan_create allocates), so this call takes the configuration and
 * computes exactly what gq_quant_error computes for it, bit for bit (cfg->workers is ignored:
 * any value is accepted, the call covers one worker's gradient).
 * Its scratch is a file-scope device array of the library, GQ_NOALLOC_SCRATCH_BYTES (about
 * 384 KB), held on every device that loads the library until the process exits.  Hence:
 *   - the input may span at most GQ_NOALLOC_MAX_BUCKETS buckets (ceil(n/d) <= 16384); larger
 *     inputs return GQ_ERR_UNSUPPORTED before anything is enqueued;
 *   - every call on a device shares that scratch and leaves its contents behind; calls whose
 *     work overlaps on the GPU (different streams or host threads) race;
 *   - there is no plan status word to query: when a kernel of the call sees a non-finite value,
 *     or a bounded wait of its kernels gives up (the kernel then stops early), all three
 *     outputs are NaN;
 *   - the first call on each device looks up the scratch's device address
 *     (cudaGetSymbolAddress) and caches it with the identity of the device's current context;
 *     make that first call, and the first call after the context was replaced (for instance by
 *     cudaDeviceReset), before any stream capture.
 * Allocates nothing, on the device or on the host.
 */
#define GQ_NOALLOC_MAX_BUCKETS 16384
#define GQ_NOALLOC_SCRATCH_BYTES (256 + 24 * (GQ_NOALLOC_MAX_BUCKETS + (GQ_NOALLOC_MAX_BUCKETS + 4095) / 4096))
GQ_API gq_status_t gq_quant_error_noalloc(const gq_config_t *cfg, uint32_t worker, uint64_t step, const float *grad,
                                          const float *residual, double *out, void *stream);

/*
 * Base-s packing of a message's codes.  The review "[Paper Review] Optimal Gradient Quantization
 * Condition for Communication-Efficient Distributed Training" ("Key findings") quotes
 * compression ratios of 20.2 for 3 levels and 10.1 for 9 levels, which are 32 / log2(s) bits:
 * codes of s levels carry log2(s) bits each, and b = ceil(log2 s) bits waste the rest.  These
 * calls convert between the dense message of gq_message_layout and a base-s message in which,
 * per bucket, g consecutive codes form one number V = sum_k code[g*i + k] * s^k (codes past the
 * bucket's d-th count as 0) of B bits:
 *     s = 3: g = 5, B = 8   (1.6 bits per code)
 *     s = 5: g = 3, B = 7   (2.33 bits per code)
 *     s = 9: g = 5, B = 16  (3.2 bits per code)
 * Other level counts return GQ_ERR_UNSUPPORTED.  Group i of a bucket is bits B*i .. B*i + B - 1,
 * least significant bit first, of the bucket's ceil(ceil(d/g) * B / 32) uint32 words (the bits
 * above the last group are 0).
 *
 * gq_entropy_layout: *bytes total; *codes_off = 0: the ceil(n/d) buckets' words, one after the
 * other; *levels_off (16-byte aligned): the level tables, exactly as in the dense message.  Host
 * computation, any output pointer may be NULL.
 */
GQ_API gq_status_t gq_entropy_layout(const gq_config_t *cfg, size_t *bytes, size_t *codes_off, size_t *levels_off);

/*
 * gq_entropy_pack: dense message -> base-s message.  gq_entropy_unpack: the inverse.
 *   cfg   the configuration the message was written with (cfg->workers is ignored).
 *   msg   device, the dense message (gq_message_layout bytes); read by pack, written completely
 *         by unpack (its padding bytes 0).
 *   emsg  device, the base-s message (gq_entropy_layout bytes); written completely by pack (its
 *         padding bytes 0), read by unpack.
 * Both 16-byte aligned and not overlapping (GQ_ERR_INVALID otherwise).  A dense message with a
 * code >= s packs to unspecified group values below 2^B, and a base-s message with a group value
 * >= s^g unpacks to unspecified codes below 2^b (accesses stay in bounds either way).
 * Stateless: no plan, no status word, no allocation; one kernel launch on `stream`.
 */
GQ_API gq_status_t gq_entropy_pack(const gq_config_t *cfg, const void *msg, void *emsg, void *stream);
GQ_API gq_status_t gq_entropy_unpack(const gq_config_t *cfg, const void *emsg, void *msg, void *stream);

/*
 * Elias-gamma coding of a message's codes.  The glossary "Gradient Quantization" (section QSGD)
 * says QSGD encodes its quantized values with Elias integer coding for further lossless
 * compression.  Elias gamma (Elias, 1975) writes x >= 1 with N = floor(log2 x) as N zero bits
 * followed by x's N + 1 bits, most significant first.  Supported: the QSGD family (QSGD,
 * TernGrad, QSGD-nearest, QSGD-l2) with an odd number of levels s and d <= 512; anything else
 * returns GQ_ERR_UNSUPPORTED.  Code c is sent as the signed level z = c - (s-1)/2, zigzag-mapped
 * to x = 2z + 1 (z >= 0) or -2z (z < 0): the zero level costs one bit.
 *
 * Message, little-endian: [uint64 T: the stream's bit count][8 zero bytes][ceil(n/d) uint64:
 * each bucket's first stream bit, padded to 16 bytes][the level tables, as in the dense message,
 * padded to 16 bytes][the stream: every bucket's valid codes in element order, stream bit k is
 * bit k % 32 of word k / 32, zero bits after T up to the next 16 bytes].  Its size depends on
 * the data: gq_elias_used_bytes(T) of the gq_elias_layout capacity are written.
 *
 * gq_elias_layout: *cap_bytes the largest message (buffers are sized for it), and the offsets of
 * the offsets region, the tables region and the stream.  Host computation; outputs may be NULL.
 * gq_elias_used_bytes: bytes of a message whose stream holds `stream_bits` bits (T, read by the
 * caller from the message's first 8 bytes).  GQ_ERR_INVALID if T exceeds the capacity.
 */
GQ_API gq_status_t gq_elias_layout(const gq_config_t *cfg, size_t *cap_bytes, size_t *offsets_off, size_t *tables_off,
                                   size_t *stream_off);
GQ_API gq_status_t gq_elias_used_bytes(const gq_config_t *cfg, uint64_t stream_bits, size_t *bytes);

/*
 * gq_elias_pack: dense message -> Elias message (five launches on `stream`; its level-table
 * region serves as the scan's scratch before the tables are written).  gq_elias_unpack: the
 * inverse (one launch).
 *   msg   device, the dense message (gq_message_layout bytes): read by pack, written completely
 *         by unpack.
 *   emsg  device, gq_elias_layout capacity bytes: its first gq_elias_used_bytes(T) bytes are
 *         written by pack (the rest is left as it was) and read by unpack.
 * Both 16-byte aligned and not overlapping (GQ_ERR_INVALID otherwise).  Codes >= s in a dense
 * message are encoded as s - 1; a damaged stream decodes to unspecified codes below 2^b, every
 * read inside the capacity.  Stateless: no plan, no allocation.
 */
GQ_API gq_status_t gq_elias_pack(const gq_config_t *cfg, const void *msg, void *emsg, void *stream);
GQ_API gq_status_t gq_elias_unpack(const gq_config_t *cfg, const void *emsg, void *msg, void *stream);

/*
 * TernGrad with one scale per parameter tensor (scheme GQ_TERNGRAD_LAYER, 3 levels).  The
 * glossary "Gradient Quantization" (section Ternary and binary quantization) gives TernGrad a
 * single scaling factor per layer; here the gradient is the concatenation of nseg tensors,
 * tensor t holding elements [offsets[t], offsets[t+1]).  Per worker m_t = max |v| over tensor t
 * (v = g + r), and each element is rounded between the two of {-m_t, 0, +m_t} around it exactly
 * as GQ_TERNGRAD rounds it (same position, probability and Philox draw).
 * Message: the 2-bit codes in the layout of the dense message (bucket after bucket), then the
 * nseg scales (float32); both regions 16-byte aligned.  gq_message_layout cannot size it (it
 * depends on nseg): use gq_plan_message_layout.
 *
 * gq_plan_set_segments: offsets is a HOST array of nseg + 1 non-decreasing offsets with
 * offsets[0] = 0 and offsets[nseg] = n (empty tensors allowed); the plan copies it to device
 * memory it owns (this call allocates, like gq_plan_create; a second call replaces the first).
 * GQ_ERR_INVALID for another scheme or bad offsets.  gq_encode, gq_decode_accumulate and
 * gq_fused_step on such a plan return GQ_ERR_INVALID until the segments are set; gq_quant_error
 * returns GQ_ERR_UNSUPPORTED.
 * gq_plan_message_layout: the plan's message size and region offsets (any scheme; for
 * GQ_TERNGRAD_LAYER once the segments are set).
 */
GQ_API gq_status_t gq_plan_set_segments(gq_plan_t plan, const int64_t *offsets, int nseg);
GQ_API gq_status_t gq_plan_message_layout(gq_plan_t plan, size_t *bytes, size_t *codes_off, size_t *levels_off);

/*
 * The format of a plan's messages.  The review "[Paper Review] Optimal Gradient Quantization
 * Condition for Communication-Efficient Distributed Training" ("Key findings") quotes compression
 * ratios of 32 / log2(s); GQ_FORMAT_BASE_S is the message of gq_entropy_pack (g codes per B-bit
 * base-s number, the level tables unchanged), written by gq_encode / gq_fused_step and read by
 * gq_decode_accumulate directly, so that no dense message exists.  s = 3, 5 or 9 levels; ORQ and
 * the QSGD family (QSGD, TernGrad, QSGD-nearest, QSGD-l2); d <= 512.
 * gq_plan_set_format: GQ_FORMAT_DENSE (the default) or GQ_FORMAT_BASE_S; afterwards
 * gq_plan_message_layout gives the message size and offsets (gq_entropy_layout's for base-s).
 * GQ_ERR_UNSUPPORTED for a plan base-s does not cover, GQ_ERR_INVALID for an unknown format.
 * Host only; no allocation.  gq_message_layout keeps describing the dense message.
 */
#define GQ_FORMAT_DENSE 0
#define GQ_FORMAT_BASE_S 1
GQ_API gq_status_t gq_plan_set_format(gq_plan_t plan, int format);

/* Synchronize `stream`, then report and clear the plan's status flags: GQ_ERR_TIMEOUT if a
 * kernel's bounded wait for a bulk copy gave up (the kernel then stopped early; its outputs are
 * incomplete), else GQ_ERR_NONFINITE if a non-finite input was seen since the last call;
 * GQ_ERR_CUDA if the stream failed. */
GQ_API gq_status_t gq_plan_status(gq_plan_t plan, void *stream);

/* Self-test of the failure path, no counterpart in the pages: every wait of the kernels for a
 * bulk copy is bounded in time and, when it gives up, raises the plan's timeout flag instead of
 * hanging.  This call enqueues one warp that waits, with the same bounded wait, on a barrier
 * that nothing completes; after limit_ns nanoseconds (clamped to [1e6, 1e9]) it raises the flag
 * and exits.  gq_plan_status then returns GQ_ERR_TIMEOUT, and the plan and the context stay
 * usable.  Returns GQ_ERR_INVALID for a NULL plan, GQ_ERR_CUDA if the launch fails. */
GQ_API gq_status_t gq_selftest_bounded_wait(gq_plan_t plan, int64_t limit_ns, void *stream);

/* Static description of a status code. */
GQ_API const char *gq_status_string(gq_status_t status);

/* Library version, "major.minor.patch". */
GQ_API const char *gq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQ_H */
