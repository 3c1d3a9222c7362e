// gq_entropy.cu -- base-s packing of a message's codes: gq_entropy_layout, gq_entropy_pack and
// gq_entropy_unpack.
//
// The review "[Paper Review] Optimal Gradient Quantization Condition for Communication-Efficient
// Distributed Training" ("Key findings") quotes compression ratios of 20.2 (3 levels) and 10.1
// (9 levels): 32 / log2(s) bits.  A code of s levels holds log2(s) bits of information, but the
// dense message stores it in b = ceil(log2 s) bits.  Here g codes of a bucket form one base-s
// number V = sum_k code[g*i + k] * s^k of B bits (s^g <= 2^B), and the group values follow each
// other in the bucket's bit string, least significant bit first.
//
// Kernel: one CTA per tile of T consecutive buckets (grid-stride over tiles).
//   1. The tile's source words are one contiguous span: 16-byte vector loads of its aligned
//      superset into shared memory (the codes region is padded to 16 bytes, so the superset
//      stays inside the message).
//   2. One thread per run of m groups (m * max(source, destination) bits <= 32): it reads the
//      run's source bits as one funnel shift of two shared words, converts each group (digits
//      of s <-> b-bit fields) and stores the run's destination bits as one shared word.
//   3. One thread per destination word: it ORs the two or three runs that overlap the word's
//      32 bits and stores it (coalesced).  The level tables are copied unchanged.
// Memory-bound: every byte of both messages is read or written once.
#include <algorithm>
#include <cstdint>

#include <nvtx3/nvToolsExt.h>

#include "gq_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kTileBytes = 24576;  // shared memory target of one tile (several CTAs per SM)

template <int S>
struct Base;
template <>
struct Base<3> {
    static constexpr int g = 5, B = 8, b = 2;
};
template <>
struct Base<5> {
    static constexpr int g = 3, B = 7, b = 3;
};
template <>
struct Base<9> {
    static constexpr int g = 5, B = 16, b = 4;
};

bool groups_for(int s, int *g, int *B, int *b)
{
    switch (s) {
    case 3: *g = Base<3>::g; *B = Base<3>::B; *b = Base<3>::b; return true;
    case 5: *g = Base<5>::g; *B = Base<5>::B; *b = Base<5>::b; return true;
    case 9: *g = Base<9>::g; *B = Base<9>::B; *b = Base<9>::b; return true;
    default: return false;
    }
}

struct EParams {
    const uint32_t *src;  // source codes region
    uint32_t *dst;        // destination codes region
    const float *tsrc;    // source level tables
    float *tdst;          // destination level tables
    int64_t nb;           // buckets
    int64_t tiles;        // ceil(nb / T)
    int d;                // bucket size
    int G;                // groups per bucket, ceil(d / g)
    int runs;             // runs of m groups per bucket, ceil(G / m)
    int sw, dw;           // source / destination words per bucket
    int T;                // buckets per tile
    int L;                // floats per level table
    // ceil(2^32 / divisor): j / divisor = umulhi(j, magic) exactly for j < 2^32 / divisor; the
    // indexes j stay below T * max(runs, dw), a few thousand (divisors are at most 10923)
    uint32_t runs_magic;  // divisor runs
    uint32_t dw_magic;    // divisor dw
    int pad_words;        // zero words after the last bucket's destination words (to 16 bytes)
    int pad_floats;       // zero floats after the last destination level table (to 16 bytes)
};

__device__ __forceinline__ uint32_t low_mask(int bits) { return bits >= 32 ? 0xffffffffu : (1u << bits) - 1u; }

// Run of M groups: source bits x (M groups of kSrc bits) -> destination bits (M groups of kDst).
template <int S, bool PACK>
struct Run {
    using C = Base<S>;
    static constexpr int kSrc = PACK ? C::b * C::g : C::B;  // source bits per group
    static constexpr int kDst = PACK ? C::B : C::b * C::g;  // destination bits per group
    static constexpr int M = 32 / (kSrc > kDst ? kSrc : kDst);
    static constexpr int kRunSrc = M * kSrc;
    static constexpr int kRunDst = M * kDst;
    static constexpr int kOverlap = 31 / kRunDst + 2;  // most runs one 32-bit word can overlap

    __device__ __forceinline__ static uint32_t convert(uint32_t x)
    {
        uint32_t out = 0;
#pragma unroll
        for (int k = 0; k < M; ++k) {
            const uint32_t grp = x >> (kSrc * k);
            uint32_t y = 0;
            if (PACK) {
                // Horner over the g b-bit codes, highest digit first
#pragma unroll
                for (int j = C::g - 1; j >= 0; --j) y = y * (uint32_t)S + ((grp >> (C::b * j)) & ((1u << C::b) - 1u));
                y &= (1u << C::B) - 1u;
            } else {
                uint32_t v = grp & ((1u << C::B) - 1u);
#pragma unroll
                for (int j = 0; j < C::g; ++j) {
                    const uint32_t q = v / (uint32_t)S;
                    y |= ((v - q * (uint32_t)S) & ((1u << C::b) - 1u)) << (C::b * j);
                    v = q;
                }
            }
            out |= y << (kDst * k);
        }
        return out;
    }
};

template <int S, bool PACK>
__global__ void __launch_bounds__(kThreads) k_entropy(const __grid_constant__ EParams p)
{
    using R = Run<S, PACK>;
    using C = Base<S>;
    extern __shared__ __align__(16) uint32_t sm[];
    const int stage_words = p.T * p.sw + 8;
    uint32_t *runs = sm + stage_words;

    if (blockIdx.x == 0) {
        if ((int)threadIdx.x < p.pad_words) p.dst[p.nb * p.dw + threadIdx.x] = 0u;
        if ((int)threadIdx.x < p.pad_floats) p.tdst[p.nb * p.L + threadIdx.x] = 0.0f;
    }

    for (int64_t tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
        const int64_t b0 = tile * p.T;
        const int nt = (int)min((int64_t)p.T, p.nb - b0);
        // 1. stage the source words [w0, w1) through their 16-byte aligned superset [a0, a1)
        const int64_t w0 = b0 * p.sw, w1 = (b0 + nt) * p.sw;
        const int64_t a0 = w0 & ~int64_t(3), a1 = (w1 + 3) & ~int64_t(3);
        const int lead = (int)(w0 - a0);
        const uint4 *src4 = reinterpret_cast<const uint4 *>(p.src + a0);
        uint4 *sm4 = reinterpret_cast<uint4 *>(sm);
        for (int v = threadIdx.x; v < (int)((a1 - a0) >> 2); v += kThreads) sm4[v] = __ldg(src4 + v);
        __syncthreads();

        // 2. runs of M groups
        const uint32_t *stage = sm + lead;
        for (int j = threadIdx.x; j < nt * p.runs; j += kThreads) {
            const int bk = (int)__umulhi((uint32_t)j, p.runs_magic);
            const int t = j - bk * p.runs;
            const uint32_t *w = stage + bk * p.sw;
            const int o = R::kRunSrc * t;
            const int q = o >> 5;
            const uint32_t lo = w[q];
            const uint32_t hi = q + 1 < p.sw ? w[q + 1] : 0u;
            uint32_t x = __funnelshift_r(lo, hi, o & 31) & low_mask(R::kRunSrc);
            if (PACK) {
                // codes past the bucket's end (the last run only) count as 0
                const int valid = p.d - C::g * R::M * t;
                if (valid < C::g * R::M) x &= (1u << (C::b * valid)) - 1u;
            }
            runs[j] = R::convert(x);
        }
        __syncthreads();

        // 3. destination words, each the OR of the runs overlapping its 32 bits
        for (int j = threadIdx.x; j < nt * p.dw; j += kThreads) {
            const int bk = (int)__umulhi((uint32_t)j, p.dw_magic);
            const int wb = j - bk * p.dw;
            const uint32_t *r = runs + bk * p.runs;
            const int lo_bit = 32 * wb;
            const int i0 = lo_bit / R::kRunDst;
            const int i1 = min((lo_bit + 31) / R::kRunDst, p.runs - 1);
            uint32_t word = 0;
#pragma unroll
            for (int k = 0; k < R::kOverlap; ++k) {
                const int i = i0 + k;
                if (i <= i1) {
                    const int sh = R::kRunDst * i - lo_bit;
                    word |= sh >= 0 ? (r[i] << sh) : (r[i] >> -sh);
                }
            }
            p.dst[b0 * p.dw + j] = word;
        }
        for (int j = threadIdx.x; j < nt * p.L; j += kThreads) p.tdst[b0 * p.L + j] = p.tsrc[b0 * p.L + j];
        __syncthreads();  // the next tile reuses the shared arrays
    }
}

struct Layouts {
    int s, g, B, b, L;
    int64_t nb;
    size_t dense_bytes, dense_levels_off;
    size_t base_bytes, base_levels_off;
    int dense_words, base_words;  // per bucket
};

int table_len(int scheme, int s)
{
    if (scheme == GQ_QSGD || scheme == GQ_TERNGRAD) return 1;
    if (scheme == GQ_BINGRAD_B || scheme == GQ_BINGRAD_PB) return 2;
    return s;
}

gq_status_t layouts(const gq_config_t *cfg, Layouts *out)
{
    if (!cfg) return GQ_ERR_INVALID;
    gq_config_t c = *cfg;
    c.workers = 1;  // ignored here
    const gq_status_t st = gq_config_check(&c);
    if (st != GQ_OK) return st;
    if (c.scheme == GQ_TERNGRAD && c.levels == 0) c.levels = 3;
    if ((c.scheme == GQ_BINGRAD_B || c.scheme == GQ_BINGRAD_PB) && c.levels == 0) c.levels = 2;
    Layouts l;
    if (!groups_for(c.levels, &l.g, &l.B, &l.b)) return GQ_ERR_UNSUPPORTED;
    size_t coff = 0;
    if (gq_message_layout(&c, &l.dense_bytes, &coff, &l.dense_levels_off) != GQ_OK) return GQ_ERR_INVALID;
    l.s = c.levels;
    l.L = table_len(c.scheme, c.levels);
    l.nb = (c.n + c.bucket - 1) / c.bucket;
    l.dense_words = c.bucket * l.b / 32;
    const int G = (c.bucket + l.g - 1) / l.g;
    l.base_words = (G * l.B + 31) / 32;
    const int64_t cbytes = (l.nb * l.base_words * 4 + 15) / 16 * 16;
    const int64_t lbytes = (l.nb * l.L * 4 + 15) / 16 * 16;
    l.base_levels_off = (size_t)cbytes;
    l.base_bytes = (size_t)(cbytes + lbytes);
    *out = l;
    return GQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int S, bool PACK>
cudaError_t launch(EParams p, cudaStream_t stream)
{
    using R = Run<S, PACK>;
    const int G = (p.d + Base<S>::g - 1) / Base<S>::g;
    p.G = G;
    p.runs = (G + R::M - 1) / R::M;
    const int per_bucket = p.sw + p.runs;  // shared words per bucket
    p.T = (int)std::max<int64_t>(1, std::min<int64_t>(p.nb, (kTileBytes / 4 - 8) / per_bucket));
    p.tiles = (p.nb + p.T - 1) / p.T;
    p.runs_magic = (uint32_t)(((uint64_t(1) << 32) + p.runs - 1) / p.runs);
    p.dw_magic = (uint32_t)(((uint64_t(1) << 32) + p.dw - 1) / p.dw);
    const size_t smem = (size_t)4 * ((size_t)p.T * p.sw + 8 + (size_t)p.T * p.runs);
    auto kern = k_entropy<S, PACK>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(p.tiles, (int64_t)sms * std::max(per_sm, 1)));
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

gq_status_t convert(const gq_config_t *cfg, const void *in, void *out, void *stream, bool pack)
{
    Layouts l;
    const gq_status_t st = layouts(cfg, &l);
    if (st != GQ_OK) return st;
    if (l.nb == 0) return GQ_OK;
    if (!in || !out || !aligned16(in) || !aligned16(out)) return GQ_ERR_INVALID;
    const size_t in_bytes = pack ? l.dense_bytes : l.base_bytes;
    const size_t out_bytes = pack ? l.base_bytes : l.dense_bytes;
    const uintptr_t i0 = reinterpret_cast<uintptr_t>(in), o0 = reinterpret_cast<uintptr_t>(out);
    if (i0 < o0 + out_bytes && o0 < i0 + in_bytes) return GQ_ERR_INVALID;

    EParams p;
    p.src = static_cast<const uint32_t *>(in);
    p.dst = static_cast<uint32_t *>(out);
    p.tsrc = reinterpret_cast<const float *>(static_cast<const unsigned char *>(in) +
                                             (pack ? l.dense_levels_off : l.base_levels_off));
    p.tdst = reinterpret_cast<float *>(static_cast<unsigned char *>(out) + (pack ? l.base_levels_off : l.dense_levels_off));
    p.nb = l.nb;
    p.d = cfg->bucket;
    p.sw = pack ? l.dense_words : l.base_words;
    p.dw = pack ? l.base_words : l.dense_words;
    p.L = l.L;
    const int64_t dst_words = l.nb * p.dw;
    p.pad_words = (int)(((dst_words + 3) & ~int64_t(3)) - dst_words);
    const int64_t tab = l.nb * l.L;
    p.pad_floats = (int)(((tab + 3) & ~int64_t(3)) - tab);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaErrorInvalidValue;
    switch (l.s) {
    case 3: e = pack ? launch<3, true>(p, s) : launch<3, false>(p, s); break;
    case 5: e = pack ? launch<5, true>(p, s) : launch<5, false>(p, s); break;
    case 9: e = pack ? launch<9, true>(p, s) : launch<9, false>(p, s); break;
    default: break;
    }
    return e == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}

struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
};

}  // namespace

extern "C" {

gq_status_t gq_entropy_layout(const gq_config_t *cfg, size_t *bytes, size_t *codes_off, size_t *levels_off)
{
    Layouts l;
    const gq_status_t st = layouts(cfg, &l);
    if (st != GQ_OK) return st;
    if (bytes) *bytes = l.base_bytes;
    if (codes_off) *codes_off = 0;
    if (levels_off) *levels_off = l.base_levels_off;
    return GQ_OK;
}

gq_status_t gq_entropy_pack(const gq_config_t *cfg, const void *msg, void *emsg, void *stream)
{
    Range range("gq_entropy_pack");
    return convert(cfg, msg, emsg, stream, true);
}

gq_status_t gq_entropy_unpack(const gq_config_t *cfg, const void *emsg, void *msg, void *stream)
{
    Range range("gq_entropy_unpack");
    return convert(cfg, emsg, msg, stream, false);
}

}  // extern "C"
