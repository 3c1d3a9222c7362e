// gq_elias.cu -- Elias-gamma coding of the codes of QSGD-family messages: gq_elias_layout,
// gq_elias_used_bytes, gq_elias_pack, gq_elias_unpack.
//
// The glossary "Gradient Quantization" (section QSGD) says that QSGD encodes its quantized
// values with Elias integer coding for further lossless compression.  Elias gamma (P. Elias,
// "Universal codeword sets and representations of the integers", 1975) writes an integer
// x >= 1 with N = floor(log2 x) as N zero bits followed by the N + 1 bits of x, most
// significant first.  With an odd number of levels s the QSGD levels include zero
// (z0 = (s-1)/2); code c becomes the signed level z = c - z0, zigzag-mapped to x = 2z + 1
// (z >= 0) or -2z (z < 0), so that the zero level costs one bit and the sparse codes of
// l2-scaled QSGD shrink to about one bit per element.
//
// Message: [T, the stream's bit count, uint64][8 zero bytes][ceil(n/d) uint64: each bucket's
// first stream bit, padded to 16 bytes][the level tables, as in the dense message, padded to
// 16 bytes][the stream: the valid codes of every bucket in element order, bit k is bit k % 32
// of word k / 32; the bits after T zero up to the next 16 bytes].
//
// Pack, five launches on the caller's stream:
//   1. k_count: one warp per bucket writes its codeword bit count into its header slot (each
//      lane over a contiguous run of codes held in a three-word register window, the next
//      bucket's window loaded one bucket ahead).
//   2. k_tile_sums: one CTA per tile of 4096 buckets sums the counts into scratch, which is
//      the message's level-table region (written last, by step 5).
//   3. k_scan_top: one CTA turns the tile sums into exclusive prefix sums, writes T, and zeroes
//      the header's second word and the stream words from the last partial one to the 16-byte
//      end.
//   4. k_scan_apply: one CTA per tile writes each bucket's first bit and zeroes the stream word
//      that a bucket shares with its predecessor.
//   5. k_encode: one warp per bucket assembles its codewords in shared memory (each lane a
//      contiguous run of elements, the run's words built in a 64-bit register), then stores
//      the words that lie wholly inside the bucket's bit range and ORs the two shared ones
//      (atomicOr on words zeroed by steps 3 and 4); the level table is copied.
// Unpack: k_decode, one thread per bucket, reads its codewords from its first bit (one table
// lookup on the next 7 bits per codeword) and writes the bucket's dense words; the level tables
// are copied.  Count and encode take each code's codeword and length from 16-entry tables.
//
// Robustness: codes >= s in a dense message are encoded as s - 1, so the stream never exceeds
// the capacity; a damaged stream decodes to unspecified codes below 2^b, with every read inside
// the message's capacity.
#include <algorithm>
#include <cstdint>

#include <nvtx3/nvToolsExt.h>

#include "gq_internal.h"

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarpThreads = 256;  // 8 warps per CTA for the per-bucket kernels
constexpr int kTile = 4096;        // buckets per scan tile
constexpr int kScanThreads = 1024; // 4 buckets per thread
constexpr int kMaxStageWords = 512 * 7 / 32 + 4;  // d <= 512, at most 7 bits per code (s <= 15)

struct ElParams {
    const uint32_t *dense;  // dense codes region
    const float *dtab;      // dense level tables
    uint64_t *hdr;          // [T, 0]
    uint64_t *offs;         // first stream bit of each bucket
    float *etab;            // level tables of the Elias message
    uint64_t *scratch;      // tile sums (inside the Elias message's level-table region)
    uint32_t *stream;
    int64_t nb, ntiles, cap_words;
    int d, s, b, L, dw, tail, z0;
    // per code c (0..15, codes >= s taken as s - 1): its codeword in stream order (the N zero
    // bits, then x most significant bit first; at most 7 bits) and its length
    unsigned long long cw_lo, cw_hi;  // 8 bits per code: codes 0..7, 8..15
    unsigned long long len_tab;       // 4 bits per code
    // decoding: the next 7 stream bits -> code | length << 4 (one byte each)
    unsigned char dec[128];
};

__device__ __forceinline__ int bucket_valid(const ElParams &p, int64_t bk) { return bk == p.nb - 1 ? p.tail : p.d; }

__device__ __forceinline__ int code_len(const ElParams &p, int c) { return (int)((p.len_tab >> (4 * c)) & 15u); }
__device__ __forceinline__ uint32_t code_word(const ElParams &p, int c)
{
    return (uint32_t)(((c < 8 ? p.cw_lo : p.cw_hi) >> (8 * (c & 7))) & 0xFFu);
}

// A lane's run of d/32 consecutive codes (at most 64 bits) in a window of three dense words
// starting at word q0 = floor(b * e0 / 32); words past the bucket's end read as 0.
struct Run {
    uint32_t w[3];
    int base;  // bit offset of code e0 inside the window
};
__device__ __forceinline__ Run load_run(const ElParams &p, const uint32_t *bw, int e0)
{
    Run r;
    const int bit = p.b * e0, q0 = bit >> 5;
#pragma unroll
    for (int k = 0; k < 3; ++k) r.w[k] = q0 + k < p.dw ? bw[q0 + k] : 0u;
    r.base = bit & 31;
    return r;
}
// code j of the run (the raw b bits; the tables map codes >= s to s - 1)
template <int B>
__device__ __forceinline__ int run_code(const Run &r, int j)
{
    const int bit = r.base + B * j;
    const uint64_t two = bit < 32 ? ((uint64_t)r.w[1] << 32) | r.w[0] : ((uint64_t)r.w[2] << 32) | r.w[1];
    return (int)((uint32_t)(two >> (bit & 31)) & ((1u << B) - 1u));
}

// ---- 1. counts ----------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kWarpThreads) k_count(const __grid_constant__ ElParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (kWarpThreads / 32);
    const int per_lane = p.d / 32, e0 = lane * per_lane;
    int64_t bk = (int64_t)blockIdx.x * (kWarpThreads / 32) + (threadIdx.x >> 5);
    Run nr{};
    if (bk < p.nb) nr = load_run(p, p.dense + bk * p.dw, e0);
    for (; bk < p.nb; bk += nwarps) {
        const Run r = nr;
        const int64_t nx = bk + nwarps;
        if (nx < p.nb) nr = load_run(p, p.dense + nx * p.dw, e0);  // one bucket ahead
        const int cnt = min(per_lane, bucket_valid(p, bk) - e0);
        int bits = 0;
        for (int j = 0; j < cnt; ++j) bits += code_len(p, run_code<B>(r, j));
        bits = __reduce_add_sync(kFull, (unsigned)bits);
        if (lane == 0) p.offs[bk] = (uint64_t)bits;
    }
}

// ---- 2-4. exclusive scan of the counts ----------------------------------------------------
__device__ __forceinline__ uint64_t warp_incl_scan(uint64_t x, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

__global__ void __launch_bounds__(kScanThreads) k_tile_sums(const __grid_constant__ ElParams p)
{
    __shared__ uint64_t red[kScanThreads / 32];
    const int64_t t0 = (int64_t)blockIdx.x * kTile;
    uint64_t s = 0;
#pragma unroll
    for (int j = 0; j < kTile / kScanThreads; ++j) {
        const int64_t bk = t0 + threadIdx.x + (int64_t)j * kScanThreads;
        if (bk < p.nb) s += p.offs[bk];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint64_t v = red[threadIdx.x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        if (threadIdx.x == 0) p.scratch[blockIdx.x] = v;
    }
}

__global__ void __launch_bounds__(kScanThreads) k_scan_top(const __grid_constant__ ElParams p)
{
    __shared__ uint64_t wsum[kScanThreads / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint64_t carry = 0;
    for (int64_t c0 = 0; c0 < p.ntiles; c0 += kScanThreads) {
        const int64_t i = c0 + threadIdx.x;
        const uint64_t x = i < p.ntiles ? p.scratch[i] : 0ull;
        const uint64_t incl = warp_incl_scan(x, lane);
        if (lane == 31) wsum[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            const uint64_t v = wsum[lane];
            wsum[lane] = warp_incl_scan(v, lane);  // inclusive over warps
        }
        __syncthreads();
        const uint64_t before = (wid > 0 ? wsum[wid - 1] : 0ull) + incl - x;
        if (i < p.ntiles) p.scratch[i] = carry + before;
        carry += wsum[kScanThreads / 32 - 1];
        __syncthreads();  // wsum is reused by the next chunk
    }
    if (threadIdx.x == 0) {
        const uint64_t T = carry;
        p.hdr[0] = T;
        p.hdr[1] = 0ull;
        if (p.nb & 1) p.offs[p.nb] = 0ull;  // padding of the offsets region
        // the last partial word and the padding words up to the 16-byte end of the stream
        const int64_t used = (int64_t)((T + 31) / 32);
        const int64_t first = (T % 32) ? used - 1 : used;
        const int64_t end = (used + 3) & ~int64_t(3);
        for (int64_t w = first; w < end && w < p.cap_words; ++w) p.stream[w] = 0u;
    }
}

__global__ void __launch_bounds__(kScanThreads) k_scan_apply(const __grid_constant__ ElParams p)
{
    __shared__ uint64_t wsum[kScanThreads / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t b0 = (int64_t)blockIdx.x * kTile + 4 * (int64_t)threadIdx.x;
    uint64_t v[4];
    uint64_t mine = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[j] = b0 + j < p.nb ? p.offs[b0 + j] : 0ull;
        mine += v[j];
    }
    const uint64_t incl = warp_incl_scan(mine, lane);
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        const uint64_t x = wsum[lane];
        wsum[lane] = warp_incl_scan(x, lane) - x;  // exclusive over warps
    }
    __syncthreads();
    uint64_t run = p.scratch[blockIdx.x] + wsum[wid] + incl - mine;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (b0 + j < p.nb) {
            p.offs[b0 + j] = run;
            if (run & 31u) p.stream[run >> 5] = 0u;  // shared with the previous bucket
        }
        run += v[j];
    }
}

// ---- 5. encode ----------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kWarpThreads) k_encode(const __grid_constant__ ElParams p, int pad_floats)
{
    __shared__ uint32_t stage_all[kWarpThreads / 32][kMaxStageWords];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    // padding of the level-table region (it held the scan's tile sums)
    if (blockIdx.x == 0 && (int)threadIdx.x < pad_floats) p.etab[p.nb * p.L + threadIdx.x] = 0.0f;
    uint32_t *st = stage_all[wid];
    const int64_t nwarps = (int64_t)gridDim.x * (kWarpThreads / 32);
    const int per_lane = p.d / 32;
    const int e0 = lane * per_lane;
    // software pipeline: the next bucket's code window, first bit and table entry are loaded
    // before this bucket is written, so the warp waits on one round trip per bucket, not three
    int64_t bk = (int64_t)blockIdx.x * (kWarpThreads / 32) + wid;
    Run nr{};
    uint64_t noff = 0;
    float ntab = 0.0f;
    if (bk < p.nb) {
        nr = load_run(p, p.dense + bk * p.dw, e0);
        noff = p.offs[bk];
        if (lane < p.L) ntab = p.dtab[bk * p.L + lane];
    }
    for (; bk < p.nb; bk += nwarps) {
        const Run rr = nr;
        const uint64_t off = noff;
        const float tab = ntab;
        const int64_t nx = bk + nwarps;
        if (nx < p.nb) {
            nr = load_run(p, p.dense + nx * p.dw, e0);
            noff = p.offs[nx];
            if (lane < p.L) ntab = p.dtab[nx * p.L + lane];
        }
        const int n = bucket_valid(p, bk);
        const int cnt = min(per_lane, n - e0);
        int bits = 0;
        for (int j = 0; j < cnt; ++j) bits += code_len(p, run_code<B>(rr, j));
        int incl = bits;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        const int total = __shfl_sync(kFull, incl, 31);
        const int base = (int)(off & 31u);
        const int nw = (base + total + 31) >> 5;
        for (int j = lane; j < nw; j += 32) st[j] = 0u;
        __syncwarp();
        if (bits > 0) {
            const int pos = base + incl - bits;  // this lane's first bit in the stage
            int wi = pos >> 5, accbits = pos & 31;
            uint64_t acc = 0;
            bool first = true;
            for (int j = 0; j < cnt; ++j) {
                const int c = run_code<B>(rr, j);
                acc |= (uint64_t)code_word(p, c) << accbits;
                accbits += code_len(p, c);
                if (accbits >= 32) {
                    if (first) atomicOr(&st[wi], (uint32_t)acc);
                    else st[wi] = (uint32_t)acc;
                    first = false;
                    ++wi;
                    acc >>= 32;
                    accbits -= 32;
                }
            }
            if (accbits > 0) atomicOr(&st[wi], (uint32_t)acc);  // may be shared with the next lane
        }
        __syncwarp();
        const int64_t w0 = (int64_t)(off >> 5);
        const uint64_t end = off + (uint64_t)total;
        for (int j = lane; j < nw; j += 32) {
            const int64_t gw = w0 + j;
            const bool whole = (uint64_t)gw * 32 >= off && (uint64_t)gw * 32 + 32 <= end;
            if (whole) p.stream[gw] = st[j];
            else atomicOr(&p.stream[gw], st[j]);
        }
        if (lane < p.L) p.etab[bk * p.L + lane] = tab;
        __syncwarp();  // the stage is reused by the next bucket
    }
}

// ---- unpack -------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t stream_word(const ElParams &p, int64_t q)
{
    return q < p.cap_words ? __ldg(p.stream + q) : 0u;
}

// One thread per bucket.  The thread reads its stream through a 64-bit bit buffer refilled a
// word at a time, with the next word's load issued one refill ahead, and decodes one codeword
// per lookup: the next 7 stream bits index a 128-entry shared table (code, length).
template <int B>
__global__ void __launch_bounds__(256) k_decode(const __grid_constant__ ElParams p, float *dtab_out,
                                                uint32_t *dense_out, int pad_floats)
{
    __shared__ unsigned char dec[128];
    if (threadIdx.x < 128) dec[threadIdx.x] = p.dec[threadIdx.x];
    __syncthreads();
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = tid; j < p.nb * p.L; j += nthreads) dtab_out[j] = p.etab[j];
    if (tid < pad_floats) dtab_out[p.nb * p.L + tid] = 0.0f;
    for (int64_t bk = tid; bk < p.nb; bk += nthreads) {
        const int n = bucket_valid(p, bk);
        uint32_t *out = dense_out + bk * p.dw;
        const uint64_t start = p.offs[bk];
        int64_t q = (int64_t)(start >> 5);
        const int sh = (int)(start & 31u);
        uint64_t buf = ((uint64_t)stream_word(p, q) | ((uint64_t)stream_word(p, q + 1) << 32)) >> sh;
        int nbuf = 64 - sh;
        q += 2;
        uint32_t next = stream_word(p, q);
        uint64_t acc = 0;
        int accbits = 0, wi = 0;
        for (int e = 0; e < n; ++e) {
            if (nbuf < 32) {  // refill: a codeword has at most 7 bits
                buf |= (uint64_t)next << nbuf;
                nbuf += 32;
                next = stream_word(p, ++q);
            }
            const unsigned t = dec[(uint32_t)buf & 127u];
            const int len = (int)(t >> 4);
            buf >>= len;
            nbuf -= len;
            acc |= (uint64_t)(t & 15u) << accbits;
            accbits += B;
            if (accbits >= 32) {
                out[wi++] = (uint32_t)acc;
                acc >>= 32;
                accbits -= 32;
            }
        }
        if (accbits > 0) out[wi++] = (uint32_t)acc;
        for (; wi < p.dw; ++wi) out[wi] = 0u;  // padding codes of a ragged last bucket
    }
}

// ---- host --------------------------------------------------------------------------------
struct ElLayout {
    int s, b, L, maxbits;
    int64_t nb;
    size_t offsets_off, tables_off, stream_off, cap;
    size_t dense_bytes, dense_levels_off;
};

int gamma_len_host(uint32_t x)
{
    int N = 0;
    while ((x >> (N + 1)) != 0u) ++N;
    return 2 * N + 1;
}

gq_status_t el_layout(const gq_config_t *cfg, ElLayout *out)
{
    if (!cfg) return GQ_ERR_INVALID;
    gq_config_t c = *cfg;
    c.workers = 1;  // ignored here
    const gq_status_t st = gq_config_check(&c);
    if (st != GQ_OK) return st;
    if (c.scheme == GQ_TERNGRAD && c.levels == 0) c.levels = 3;
    const bool qs = c.scheme == GQ_QSGD || c.scheme == GQ_TERNGRAD || c.scheme == GQ_QSGD_NEAREST ||
                    c.scheme == GQ_QSGD_L2;
    if (!qs || c.levels % 2 == 0 || c.levels > 15 || c.bucket > 512) return GQ_ERR_UNSUPPORTED;
    ElLayout l;
    l.s = c.levels;
    l.b = 0;
    while ((1 << l.b) < l.s) ++l.b;
    l.L = 1;
    l.maxbits = gamma_len_host((uint32_t)l.s);
    l.nb = (c.n + c.bucket - 1) / c.bucket;
    size_t coff = 0;
    if (gq_message_layout(&c, &l.dense_bytes, &coff, &l.dense_levels_off) != GQ_OK) return GQ_ERR_INVALID;
    const int64_t obytes = (l.nb * 8 + 15) / 16 * 16;
    const int64_t tbytes = (l.nb * l.L * 4 + 15) / 16 * 16;
    const int64_t sbytes = ((c.n * l.maxbits + 31) / 32 * 4 + 15) / 16 * 16;
    l.offsets_off = 16;
    l.tables_off = 16 + (size_t)obytes;
    l.stream_off = l.tables_off + (size_t)tbytes;
    l.cap = l.stream_off + (size_t)sbytes;
    *out = l;
    return GQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ElParams make_params(const gq_config_t *cfg, const ElLayout &l, const void *msg, const void *emsg)
{
    ElParams p;
    const unsigned char *m = static_cast<const unsigned char *>(msg);
    unsigned char *e = static_cast<unsigned char *>(const_cast<void *>(emsg));
    p.dense = reinterpret_cast<const uint32_t *>(m);
    p.dtab = reinterpret_cast<const float *>(m + l.dense_levels_off);
    p.hdr = reinterpret_cast<uint64_t *>(e);
    p.offs = reinterpret_cast<uint64_t *>(e + l.offsets_off);
    p.etab = reinterpret_cast<float *>(e + l.tables_off);
    p.scratch = reinterpret_cast<uint64_t *>(e + l.tables_off);
    p.stream = reinterpret_cast<uint32_t *>(e + l.stream_off);
    p.nb = l.nb;
    p.ntiles = (l.nb + kTile - 1) / kTile;
    p.cap_words = (int64_t)((l.cap - l.stream_off) / 4);
    p.d = cfg->bucket;
    p.s = l.s;
    p.b = l.b;
    p.L = l.L;
    p.dw = cfg->bucket * l.b / 32;
    p.tail = (int)(cfg->n - (l.nb - 1) * (int64_t)cfg->bucket);
    p.z0 = (l.s - 1) / 2;
    // codeword tables: code c -> z = c - z0 -> x = 2z + 1 (z >= 0) or -2z (z < 0) -> N zero bits,
    // then x's N + 1 bits most significant first (stream order: first bit in bit 0)
    p.cw_lo = p.cw_hi = p.len_tab = 0ull;
    for (int c = 0; c < 16; ++c) {
        const int cc = std::min(c, l.s - 1);
        const int z = cc - p.z0;
        const uint32_t x = z >= 0 ? (uint32_t)(2 * z + 1) : (uint32_t)(-2 * z);
        int N = 0;
        while ((x >> (N + 1)) != 0u) ++N;
        uint32_t v = 0;
        for (int j = 0; j <= N; ++j)  // bit N - j of x goes to stream position N + j
            if ((x >> (N - j)) & 1u) v |= 1u << (N + j);
        const unsigned long long vv = (unsigned long long)v << (8 * (c & 7));
        if (c < 8) p.cw_lo |= vv;
        else p.cw_hi |= vv;
        p.len_tab |= (unsigned long long)(2 * N + 1) << (4 * c);
    }
    // decoding table over the next 7 stream bits (a codeword here has at most 7 bits); a bit
    // pattern that starts no valid codeword decodes to code s - 1 and consumes 7 bits
    for (int t = 0; t < 128; ++t) {
        int N = 0;
        while (N < 7 && !((t >> N) & 1)) ++N;
        int code = l.s - 1, len = 7;
        if (2 * N + 1 <= 7) {
            uint32_t x = 0;
            for (int j = 0; j <= N; ++j) x = (x << 1) | (uint32_t)((t >> (N + j)) & 1);
            const int z = (x & 1u) ? (int)((x - 1u) / 2u) : -(int)(x / 2u);
            code = std::min(std::max(z + p.z0, 0), (1 << l.b) - 1);
            len = 2 * N + 1;
        }
        p.dec[t] = (unsigned char)(code | (len << 4));
    }
    return p;
}

int warp_grid(int64_t nb)
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    const int64_t want = (nb + kWarpThreads / 32 - 1) / (kWarpThreads / 32);
    return (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * (2048 / kWarpThreads)));
}

struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
};

}  // namespace

extern "C" {

gq_status_t gq_elias_layout(const gq_config_t *cfg, size_t *cap_bytes, size_t *offsets_off, size_t *tables_off,
                            size_t *stream_off)
{
    ElLayout l;
    const gq_status_t st = el_layout(cfg, &l);
    if (st != GQ_OK) return st;
    if (cap_bytes) *cap_bytes = l.cap;
    if (offsets_off) *offsets_off = l.offsets_off;
    if (tables_off) *tables_off = l.tables_off;
    if (stream_off) *stream_off = l.stream_off;
    return GQ_OK;
}

gq_status_t gq_elias_used_bytes(const gq_config_t *cfg, uint64_t stream_bits, size_t *bytes)
{
    ElLayout l;
    const gq_status_t st = el_layout(cfg, &l);
    if (st != GQ_OK) return st;
    if (!bytes) return GQ_ERR_INVALID;
    if (stream_bits > (uint64_t)(l.cap - l.stream_off) * 8) return GQ_ERR_INVALID;
    *bytes = l.stream_off + (size_t)(((stream_bits + 31) / 32 * 4 + 15) / 16 * 16);
    return GQ_OK;
}

gq_status_t gq_elias_pack(const gq_config_t *cfg, const void *msg, void *emsg, void *stream)
{
    Range range("gq_elias_pack");
    ElLayout l;
    const gq_status_t st = el_layout(cfg, &l);
    if (st != GQ_OK) return st;
    if (l.nb == 0) return GQ_OK;
    if (!msg || !emsg || !aligned16(msg) || !aligned16(emsg)) return GQ_ERR_INVALID;
    const uintptr_t i0 = reinterpret_cast<uintptr_t>(msg), o0 = reinterpret_cast<uintptr_t>(emsg);
    if (i0 < o0 + l.cap && o0 < i0 + l.dense_bytes) return GQ_ERR_INVALID;
    const ElParams p = make_params(cfg, l, msg, emsg);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int g = warp_grid(l.nb);
    auto count = l.b == 2 ? k_count<2> : l.b == 3 ? k_count<3> : k_count<4>;
    auto encode = l.b == 2 ? k_encode<2> : l.b == 3 ? k_encode<3> : k_encode<4>;
    count<<<g, kWarpThreads, 0, s>>>(p);
    k_tile_sums<<<(unsigned)p.ntiles, kScanThreads, 0, s>>>(p);
    k_scan_top<<<1, kScanThreads, 0, s>>>(p);
    k_scan_apply<<<(unsigned)p.ntiles, kScanThreads, 0, s>>>(p);
    const int64_t tab = l.nb * l.L;
    encode<<<g, kWarpThreads, 0, s>>>(p, (int)(((tab + 3) & ~int64_t(3)) - tab));
    return cudaGetLastError() == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}

gq_status_t gq_elias_unpack(const gq_config_t *cfg, const void *emsg, void *msg, void *stream)
{
    Range range("gq_elias_unpack");
    ElLayout l;
    const gq_status_t st = el_layout(cfg, &l);
    if (st != GQ_OK) return st;
    if (l.nb == 0) return GQ_OK;
    if (!msg || !emsg || !aligned16(msg) || !aligned16(emsg)) return GQ_ERR_INVALID;
    const uintptr_t i0 = reinterpret_cast<uintptr_t>(emsg), o0 = reinterpret_cast<uintptr_t>(msg);
    if (i0 < o0 + l.dense_bytes && o0 < i0 + l.cap) return GQ_ERR_INVALID;
    const ElParams p = make_params(cfg, l, msg, emsg);
    unsigned char *m = static_cast<unsigned char *>(msg);
    const int64_t tab = l.nb * l.L;
    const int pad = (int)(((tab + 3) & ~int64_t(3)) - tab);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((l.nb + 255) / 256, (int64_t)sms * 8));
    auto decode = l.b == 2 ? k_decode<2> : l.b == 3 ? k_decode<3> : k_decode<4>;
    decode<<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        p, reinterpret_cast<float *>(m + l.dense_levels_off), reinterpret_cast<uint32_t *>(m), pad);
    return cudaGetLastError() == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}

}  // extern "C"
