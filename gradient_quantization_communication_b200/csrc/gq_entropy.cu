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
//   1. The tile's source words are one contiguous span: 16-byte asynchronous copies (cp.async)
//      of its aligned superset into shared memory (the codes region is padded to 16 bytes, so
//      the superset stays inside the message), issued one tile ahead into a second buffer.
//   2. One thread per chunk (a run of groups that starts on a word in both bit strings, see
//      gq_entropy.cuh): it reads the chunk's source words from shared memory (words past the
//      bucket's end as 0), converts them in registers and stores its destination words to a
//      second shared array.
//   3. The tile's destination words are again one contiguous span: coalesced stores.  The level
//      tables are copied unchanged.
// Memory-bound by design: every byte of both messages is read or written once.
#include <algorithm>
#include <atomic>
#include <cstdint>

#include <nvtx3/nvToolsExt.h>

#include "gq_entropy.cuh"
#include "gq_internal.h"

namespace {

using gq::entropy::Base;
using gq::entropy::Chunk;

constexpr int kThreads = 256;
constexpr int kTileBytes = 24576;  // shared memory target of one CTA (8 CTAs of 256 threads per SM)
constexpr int kTabRegs = 4;        // level-table floats per thread and tile: T * L <= 4 * kThreads

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
    int chunks;           // chunks per bucket
    int sw, dw;           // source / destination words per bucket
    int T;                // buckets per tile
    int L;                // floats per level table
    // ceil(2^32 / chunks): j / chunks = umulhi(j, magic) exactly for j < 2^32 / chunks; the
    // indexes j stay below T * chunks, a few thousand
    uint32_t chunks_magic;
    int stage_words;      // words of one source buffer in shared memory (a multiple of 4)
    int pad_words;        // zero words after the last bucket's destination words (to 16 bytes)
    int pad_floats;       // zero floats after the last destination level table (to 16 bytes)
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// waits until at most N of this thread's committed groups are still in flight (the hardware
// completes every issued copy; nothing here spins)
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Source words of tile `tile`: buckets [b0, b0 + nt), words [w0, w1) of the source codes,
// copied through their 16-byte aligned superset [a0, a1) (inside the padded codes region).
struct TileSpan {
    int64_t b0, a0;
    int nt, lead, nvec;
};
__device__ __forceinline__ TileSpan tile_span(const EParams &p, int64_t tile)
{
    TileSpan t;
    t.b0 = tile * p.T;
    t.nt = (int)min((int64_t)p.T, p.nb - t.b0);
    const int64_t w0 = t.b0 * p.sw, w1 = (t.b0 + t.nt) * p.sw;
    t.a0 = w0 & ~int64_t(3);
    t.lead = (int)(w0 - t.a0);
    t.nvec = (int)((((w1 + 3) & ~int64_t(3)) - t.a0) >> 2);
    return t;
}

__device__ __forceinline__ void stage_tile(const EParams &p, const TileSpan &t, uint32_t *buf)
{
    for (int v = threadIdx.x; v < t.nvec; v += kThreads) cp_async16(buf + 4 * v, p.src + t.a0 + 4 * v);
}

template <int S, bool PACK>
__global__ void __launch_bounds__(kThreads) k_entropy(const __grid_constant__ EParams p)
{
    using K = Chunk<S, PACK>;
    extern __shared__ __align__(16) uint32_t sm[];
    // [source buffer 0 | source buffer 1 | destination words], each 16-byte aligned: the next
    // tile's source words are copied in (cp.async) while this tile is converted
    uint32_t *out = sm + 2 * p.stage_words;

    if (blockIdx.x == 0) {
        if ((int)threadIdx.x < p.pad_words) p.dst[p.nb * p.dw + threadIdx.x] = 0u;
        if ((int)threadIdx.x < p.pad_floats) p.tdst[p.nb * p.L + threadIdx.x] = 0.0f;
    }

    int64_t tile = blockIdx.x;
    if (tile < p.tiles) stage_tile(p, tile_span(p, tile), sm);
    cp_async_commit();
    for (int it = 0; tile < p.tiles; tile += gridDim.x, ++it) {
        const TileSpan t = tile_span(p, tile);
        const int64_t next = tile + gridDim.x;
        if (next < p.tiles) stage_tile(p, tile_span(p, next), sm + ((it & 1) ? 0 : p.stage_words));
        cp_async_commit();
        // this tile's level tables into registers; their latency overlaps the conversion
        float tv[kTabRegs];
#pragma unroll
        for (int k = 0; k < kTabRegs; ++k) {
            const int j = threadIdx.x + k * kThreads;
            tv[k] = j < t.nt * p.L ? p.tsrc[t.b0 * p.L + j] : 0.0f;
        }
        cp_async_wait<1>();  // this tile's copies (all but the group just committed)
        __syncthreads();

        // one chunk per thread.  The destination words start at `o` + 0, placed so that o and
        // the tile's first destination word in global memory agree modulo 16 bytes.
        const uint32_t *stage = sm + ((it & 1) ? p.stage_words : 0) + t.lead;
        const int off = (int)((t.b0 * p.dw) & 3);
        uint32_t *o = out + off;
        for (int j = threadIdx.x; j < t.nt * p.chunks; j += kThreads) {
            const int bk = (int)__umulhi((uint32_t)j, p.chunks_magic);
            const int c = j - bk * p.chunks;
            const int s0 = c * K::kSrcWords, d0 = c * K::kDstWords;
            const uint32_t *w = stage + bk * p.sw + s0;
            uint32_t *ow = o + bk * p.dw + d0;
            // words past the bucket's end (its last chunk only) read as 0 and are not written;
            // one predicated path for all chunks, so that the lanes of a warp do not diverge
            uint32_t in[K::kSrcWords], res[K::kDstWords];
#pragma unroll
            for (int k = 0; k < K::kSrcWords; ++k) in[k] = s0 + k < p.sw ? w[k] : 0u;
            gq::entropy::convert_chunk<S, PACK>(in, res);
#pragma unroll
            for (int k = 0; k < K::kDstWords; ++k)
                if (d0 + k < p.dw) ow[k] = res[k];
        }
        __syncthreads();

        // the tile's destination words (one contiguous span: scalar head and tail, 16-byte
        // body) and level tables
        uint32_t *dst = p.dst + t.b0 * p.dw;
        const int nw = t.nt * p.dw;
        const int head = min((4 - off) & 3, nw);
        const int nvec = (nw - head) >> 2;
        const int tail0 = head + 4 * nvec;
        if ((int)threadIdx.x < head) dst[threadIdx.x] = o[threadIdx.x];
        {
            const uint4 *o4 = reinterpret_cast<const uint4 *>(o + head);
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + head);
            for (int j = threadIdx.x; j < nvec; j += kThreads) d4[j] = o4[j];
        }
        if ((int)threadIdx.x < nw - tail0) dst[tail0 + threadIdx.x] = o[tail0 + threadIdx.x];
#pragma unroll
        for (int k = 0; k < kTabRegs; ++k) {
            const int j = threadIdx.x + k * kThreads;
            if (j < t.nt * p.L) p.tdst[t.b0 * p.L + j] = tv[k];
        }
        // the next iteration's first __syncthreads orders these reads of `out` before its writes,
        // and this iteration's second one ordered the reads of this tile's buffer before the
        // copies into it that the next iteration issues
    }
    cp_async_wait<0>();
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
    if (scheme == GQ_QSGD || scheme == GQ_TERNGRAD || scheme == GQ_QSGD_NEAREST || scheme == GQ_QSGD_L2) return 1;
    if (scheme == GQ_BINGRAD_B || scheme == GQ_BINGRAD_PB || scheme == GQ_SIGNSGD) return 2;
    return s;
}

gq_status_t layouts(const gq_config_t *cfg, Layouts *out)
{
    if (!cfg) return GQ_ERR_INVALID;
    gq_config_t c = *cfg;
    c.workers = 1;  // ignored here
    const gq_status_t st = gq_config_check(&c);
    if (st != GQ_OK) return st;
    if (c.scheme == GQ_TERNGRAD_LAYER) return GQ_ERR_UNSUPPORTED;  // its message holds per-tensor scales
    if (c.scheme == GQ_TERNGRAD && c.levels == 0) c.levels = 3;
    if ((c.scheme == GQ_BINGRAD_B || c.scheme == GQ_BINGRAD_PB || c.scheme == GQ_SIGNSGD) && c.levels == 0)
        c.levels = 2;
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
cudaError_t launch(EParams p, int d, cudaStream_t stream)
{
    using C = Base<S>;
    const int G = (d + C::g - 1) / C::g;
    p.chunks = (G + C::CG - 1) / C::CG;
    const int per_bucket = 2 * p.sw + p.dw;  // shared words per bucket
    int64_t T = std::min<int64_t>(p.nb, (kTileBytes / 4 - 28) / per_bucket);
    T = std::min<int64_t>(T, kTabRegs * kThreads / p.L);
    // whole passes of the CTA's threads over the tile's chunks (no near-empty last pass)
    if (T * p.chunks >= kThreads) T = (T * p.chunks / kThreads) * kThreads / p.chunks;
    p.T = (int)std::max<int64_t>(1, T);
    p.tiles = (p.nb + p.T - 1) / p.T;
    p.chunks_magic = (uint32_t)(((uint64_t(1) << 32) + p.chunks - 1) / p.chunks);
    // [2 x (source words of a tile + up to 3 + 3 of alignment) | up to 3 + destination words
    // of a tile]
    p.stage_words = (p.T * p.sw + 8 + 3) & ~3;
    const size_t smem = (size_t)4 * (2 * (size_t)p.stage_words + 3 + (size_t)p.T * p.dw);
    auto kern = k_entropy<S, PACK>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    // the whole unified L1 as shared memory: eight CTAs of ~23 KB per SM (the kernel reads
    // global memory only through the asynchronous copies and the level tables)
    static std::atomic<bool> carveout_set{false};  // a repeated set is harmless, so no lock
    if (!carveout_set.load(std::memory_order_relaxed)) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                                   (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        carveout_set.store(true, std::memory_order_relaxed);
    }
    // grid-stride over tiles: at most as many CTAs as fit on the device at full occupancy
    // (2048 threads per SM); with less shared memory per SM some wait for a free slot
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(p.tiles, (int64_t)sms * (2048 / kThreads)));
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
    case 3: e = pack ? launch<3, true>(p, cfg->bucket, s) : launch<3, false>(p, cfg->bucket, s); break;
    case 5: e = pack ? launch<5, true>(p, cfg->bucket, s) : launch<5, false>(p, cfg->bucket, s); break;
    case 9: e = pack ? launch<9, true>(p, cfg->bucket, s) : launch<9, false>(p, cfg->bucket, s); break;
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
