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
//   1. k_count: one thread per bucket writes its codeword bit count into its header slot; a warp
//      copies its 32 buckets' dense words into shared rows with coalesced loads first, and each
//      thread walks its row G codes per table lookup.
//   2. k_tile_sums: one CTA per tile of 4096 buckets sums the counts into scratch, which is
//      the message's level-table region (written last, by step 5).
//   3. k_scan_top: one CTA turns the tile sums into exclusive prefix sums, writes T, and zeroes
//      the header's second word and the stream words from the last partial one to the 16-byte
//      end.
//   4. k_scan_apply: one CTA per tile writes each bucket's first bit and zeroes the stream word
//      that a bucket shares with its predecessor.
//   5. k_encode: one thread per bucket (rows as in step 1) appends its codewords, G codes per
//      table lookup, to a 64-bit bit buffer aligned to its first stream bit and stores each full
//      word; the words it shares with its neighbours (the first and the last, when the bucket
//      starts or ends inside a word) go by atomicOr onto words zeroed by steps 3 and 4; the level
//      table is copied.
// Unpack: k_decode, one thread per bucket, reads its codewords from its first bit (one lookup of
// the next 10 bits decodes every codeword inside them) into the warp's shared rows, and the warp
// writes 32 buckets' dense words at a time; the level tables are copied.  Count and encode take
// the codewords and lengths of 2 or 4 codes at once from 256-entry tables.
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
constexpr int kTile = 4096;        // buckets per scan tile
constexpr int kScanThreads = 1024; // 4 buckets per thread

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
    // G = 8 / b codes (2 for b = 3) as one table index of G * b bits -> their codewords in stream
    // order (bits 0 .. 23) | total length << 24
    uint32_t enc[256];
};

// codes per table index of the group tables
template <int B>
__host__ __device__ constexpr int group_codes() { return B == 3 ? 2 : 8 / B; }

__device__ __forceinline__ int bucket_valid(const ElParams &p, int64_t bk) { return bk == p.nb - 1 ? p.tail : p.d; }

__device__ __forceinline__ int code_len(const ElParams &p, int c) { return (int)((p.len_tab >> (4 * c)) & 15u); }
__device__ __forceinline__ uint32_t code_word(const ElParams &p, int c)
{
    return (uint32_t)(((c < 8 ? p.cw_lo : p.cw_hi) >> (8 * (c & 7))) & 0xFFu);
}

// ---- 1. counts ----------------------------------------------------------------------------
// One thread per bucket, a warp per 32 consecutive buckets: the warp copies the 32 buckets'
// dense words (one contiguous span) into its shared rows with coalesced loads, then each thread
// walks its row by table index (G codes at a time).
constexpr int kBktWarps = 4;  // warps per CTA of the thread-per-bucket kernels

// Group k (G codes, G * B bits) of a row of dense words.
template <int B>
__device__ __forceinline__ uint32_t row_group(const uint32_t *row, int k)
{
    constexpr int G = group_codes<B>(), NB = G * B;
    if constexpr (NB == 8) {
        return (row[k >> 2] >> (8 * (k & 3))) & 0xFFu;
    } else {
        const int bit = NB * k, w = bit >> 5, sh = bit & 31;
        const uint32_t lo = row[w] >> sh;
        const uint32_t hi = sh + NB > 32 ? row[w + 1] << (32 - sh) : 0u;
        return (lo | hi) & ((1u << NB) - 1u);
    }
}
// Code j of a row of dense words.
template <int B>
__device__ __forceinline__ int row_code(const uint32_t *row, int j)
{
    const int bit = B * j, w = bit >> 5, sh = bit & 31;
    uint32_t x = row[w] >> sh;
    if (sh + B > 32) x |= row[w + 1] << (32 - sh);
    return (int)(x & ((1u << B) - 1u));
}

// The warp's 32 buckets from bk0 into rows [32][dw + 1] (the pad word stays 0).  The buckets'
// words are one contiguous span (dw is a multiple of 4): 16-byte loads, eight in flight per lane
// before any is stored.
__device__ __forceinline__ void load_rows(const ElParams &p, uint32_t *rows, int64_t bk0, int lane)
{
    const int dw = p.dw, rs = p.dw + 1;
    const int nrows = (int)min((int64_t)32, p.nb - bk0);
    const uint4 *src = reinterpret_cast<const uint4 *>(p.dense + bk0 * dw);
    const int nq = nrows * dw / 4;
    for (int i0 = 0; i0 < nq; i0 += 8 * 32) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + 32 * u + lane;
            if (i < nq) v[u] = __ldg(src + i);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + 32 * u + lane;
            if (i < nq) {
                const int w = 4 * i, r = w / dw, c = w - r * dw;
                uint32_t *d = rows + r * rs + c;
                d[0] = v[u].x;
                d[1] = v[u].y;
                d[2] = v[u].z;
                d[3] = v[u].w;
            }
        }
    }
    if (lane < nrows) rows[lane * rs + dw] = 0u;
}

template <int B>
__global__ void __launch_bounds__(kBktWarps * 32) k_count(const __grid_constant__ ElParams p)
{
    constexpr int G = group_codes<B>();
    __shared__ uint32_t enc[256];
    extern __shared__ uint32_t rows_all[];  // [warps][32][dw + 1]
    for (int i = threadIdx.x; i < (1 << (G * B)); i += blockDim.x) enc[i] = p.enc[i];
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int rs = p.dw + 1;
    uint32_t *rows = rows_all + wid * 32 * rs;
    const uint32_t *row = rows + lane * rs;
    const int64_t nwarps = (int64_t)gridDim.x * kBktWarps;
    for (int64_t bk0 = ((int64_t)blockIdx.x * kBktWarps + wid) * 32; bk0 < p.nb; bk0 += nwarps * 32) {
        load_rows(p, rows, bk0, lane);
        __syncwarp();
        const int64_t bk = bk0 + lane;
        if (bk < p.nb) {
            const int n = bucket_valid(p, bk);
            const int ng = n / G;
            int bits = 0, k = 0;
            if constexpr (G * B == 8) {
                // a row word holds four whole table indices
                for (; k + 4 <= ng; k += 4) {
                    const uint32_t x = row[k >> 2];
                    bits += (int)((enc[x & 0xFFu] >> 24) + (enc[(x >> 8) & 0xFFu] >> 24) +
                                  (enc[(x >> 16) & 0xFFu] >> 24) + (enc[x >> 24] >> 24));
                }
            }
            for (; k < ng; ++k) bits += (int)(enc[row_group<B>(row, k)] >> 24);
            for (int j = ng * G; j < n; ++j) bits += code_len(p, row_code<B>(row, j));
            p.offs[bk] = (uint64_t)bits;
        }
        __syncwarp();
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
// One thread per bucket (rows as in the count): the thread appends its codewords, G codes per
// table lookup, to a 64-bit bit buffer that starts at its bucket's first stream bit and stores
// each full word.  The first word is shared with the previous bucket when the bucket starts
// inside a word, the last with the next one when it ends inside one: those go by atomicOr onto
// the words the scan zeroed; every other word belongs to this bucket alone.
template <int B>
__global__ void __launch_bounds__(kBktWarps * 32) k_encode(const __grid_constant__ ElParams p, int pad_floats)
{
    constexpr int G = group_codes<B>();
    __shared__ uint32_t enc[256];
    extern __shared__ uint32_t rows_all[];
    for (int i = threadIdx.x; i < (1 << (G * B)); i += blockDim.x) enc[i] = p.enc[i];
    __syncthreads();
    // padding of the level-table region (it held the scan's tile sums)
    if (blockIdx.x == 0 && (int)threadIdx.x < pad_floats) p.etab[p.nb * p.L + threadIdx.x] = 0.0f;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int rs = p.dw + 1;
    uint32_t *rows = rows_all + wid * 32 * rs;
    const uint32_t *row = rows + lane * rs;
    const int64_t nwarps = (int64_t)gridDim.x * kBktWarps;
    for (int64_t bk0 = ((int64_t)blockIdx.x * kBktWarps + wid) * 32; bk0 < p.nb; bk0 += nwarps * 32) {
        load_rows(p, rows, bk0, lane);
        __syncwarp();
        const int64_t bk = bk0 + lane;
        if (bk < p.nb) {
            const int n = bucket_valid(p, bk);
            const int ng = n / G;
            const uint64_t off = p.offs[bk];
            uint32_t *wp = p.stream + (off >> 5);
            int accbits = (int)(off & 31u);
            bool shared_first = accbits != 0;
            uint64_t acc = 0;
            auto flush = [&]() {
                if (shared_first) atomicOr(wp, (uint32_t)acc);
                else *wp = (uint32_t)acc;
                shared_first = false;
                ++wp;
                acc >>= 32;
                accbits -= 32;
            };
            const auto put = [&](uint32_t e) {
                acc |= (uint64_t)(e & 0xFFFFFFu) << accbits;
                accbits += (int)(e >> 24);
            };
            int k = 0;
            if constexpr (G * B == 8) {
                // a row word holds four whole table indices; two groups take at most 28 bits
                // (4 codewords of at most 3 bits, or 2 of at most 7), so one check after each pair
                // keeps the buffer below 64 bits
                for (; k + 4 <= ng; k += 4) {
                    const uint32_t x = row[k >> 2];
                    put(enc[x & 0xFFu]);
                    put(enc[(x >> 8) & 0xFFu]);
                    if (accbits >= 32) flush();
                    put(enc[(x >> 16) & 0xFFu]);
                    put(enc[x >> 24]);
                    if (accbits >= 32) flush();
                }
            }
            for (; k < ng; ++k) {
                put(enc[row_group<B>(row, k)]);
                if (accbits >= 32) flush();
            }
            for (int j = ng * G; j < n; ++j) {
                const int c = row_code<B>(row, j);
                acc |= (uint64_t)code_word(p, c) << accbits;
                accbits += code_len(p, c);
                if (accbits >= 32) flush();
            }
            if (accbits > 0) atomicOr(wp, (uint32_t)acc);  // may be shared with the next bucket
            if (p.L > 0) {
                for (int k = 0; k < p.L; ++k) p.etab[bk * p.L + k] = p.dtab[bk * p.L + k];
            }
        }
        __syncwarp();
    }
}

// ---- unpack -------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t stream_word(const ElParams &p, int64_t q)
{
    return q < p.cap_words ? __ldg(p.stream + q) : 0u;
}

// Decode CTAs: eight warps, each staging up to 2.4 KB of stream; with the window table and the
// 32 rows of dense words this keeps 32 warps resident per SM at d = 512, 2-bit codes.
constexpr int kDecodeWarps = 8;
constexpr int kStreamStage = 600;  // stream words a warp stages for its 32 buckets
// Multi-codeword lookups read the next kDecWin stream bits: the codewords that lie wholly inside
// them, decoded, as one 32-bit entry (codes b bits each at bits 0 .. 23, count << 24, bits
// consumed << 28).  At most 24 / b codes go in one entry.
constexpr int kDecWin = 10;
static_assert(3 * kDecWin <= 32, "three lookups per refill");

// The window table from the single-codeword table dec (the next 7 bits -> code | length << 4):
// decode as dec does while the next codeword lies wholly inside the window; the first one always
// does (a codeword has at most 7 bits, and a pattern that starts none takes 7).  dec saw zeros
// past the window, so its answer stands only for a codeword whose bits all lie inside.
template <int B>
__device__ __forceinline__ void build_window_table(const unsigned char *dec, uint32_t *decw)
{
    constexpr int cap = 24 / B;
    for (int t = threadIdx.x; t < (1 << kDecWin); t += blockDim.x) {
        int pos = 0, cnt = 0;
        uint32_t codes = 0;
        while (pos < kDecWin && cnt < cap) {
            const unsigned e = dec[(t >> pos) & 127];
            const int len = (int)(e >> 4);
            if (pos + len > kDecWin) break;
            codes |= (e & 15u) << (B * cnt);
            ++cnt;
            pos += len;
        }
        decw[t] = codes | ((uint32_t)cnt << 24) | ((uint32_t)pos << 28);
    }
}

// The codes of one bucket from its first stream bit: rd(q) reads stream word q.
template <int B, class Rd>
__device__ __forceinline__ void decode_bucket(const unsigned char *dec, const uint32_t *decw, uint64_t start, int n,
                                              int dw, uint32_t *out, const Rd &rd)
{
    int64_t q = (int64_t)(start >> 5);
    const int sh = (int)(start & 31u);
    uint64_t buf = ((uint64_t)rd(q) | ((uint64_t)rd(q + 1) << 32)) >> sh;
    int nbuf = 64 - sh;
    q += 2;
    uint32_t next = rd(q);
    uint64_t acc = 0;
    int accbits = 0, wi = 0;
    int e = 0;
    const auto look = [&]() {
        const uint32_t t = decw[(uint32_t)buf & ((1u << kDecWin) - 1u)];
        const int cnt = (int)((t >> 24) & 15u), len = (int)(t >> 28);
        buf >>= len;
        nbuf -= len;
        acc |= (uint64_t)(t & 0xFFFFFFu) << accbits;
        accbits += B * cnt;
        e += cnt;
        if (accbits >= 32) {
            out[wi++] = (uint32_t)acc;
            acc >>= 32;
            accbits -= 32;
        }
    };
    // a refill leaves at least 32 bits in the buffer: three lookups of up to kDecWin bits each
    for (; e + 3 * kDecWin <= n;) {
        if (nbuf < 32) {
            buf |= (uint64_t)next << nbuf;
            nbuf += 32;
            next = rd(++q);
        }
        look();
        look();
        look();
    }
    for (; e + kDecWin <= n;) {
        if (nbuf < 32) {
            buf |= (uint64_t)next << nbuf;
            nbuf += 32;
            next = rd(++q);
        }
        look();
    }
    for (; e < n; ++e) {
        if (nbuf < 32) {  // refill: a codeword has at most 7 bits
            buf |= (uint64_t)next << nbuf;
            nbuf += 32;
            next = rd(++q);
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
    for (; wi < dw; ++wi) out[wi] = 0u;  // padding codes of a ragged last bucket
}

// One thread per bucket, a warp per 32 consecutive buckets.  Their stream bits are one span:
// when it fits in kStreamStage words the warp first copies it into shared memory with coalesced
// loads, else the threads read global memory.  A thread reads its codewords through a 64-bit
// bit buffer; while at least kDecWin codes remain, one lookup of the next kDecWin stream bits
// decodes every codeword that lies wholly inside them (decw, built by each CTA), the rest go one
// codeword per lookup of the next 7 bits (dec).  The thread builds its bucket's dense words in its row of the warp's shared
// buffer (rows of dw + 1 words, so that the lanes' stores hit distinct banks); the warp then
// writes the 32 buckets' words, which are contiguous in the dense message, row by row with
// coalesced stores.
template <int B>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_decode(const __grid_constant__ ElParams p, float *dtab_out,
                                                              uint32_t *dense_out, int pad_floats)
{
    __shared__ unsigned char dec[128];
    __shared__ uint32_t decw[1 << kDecWin];
    __shared__ uint32_t stage_all[kDecodeWarps][kStreamStage];
    extern __shared__ uint32_t rows_all[];  // [warps][32][dw + 1]
    if (threadIdx.x < 128) dec[threadIdx.x] = p.dec[threadIdx.x];
    __syncthreads();
    build_window_table<B>(dec, decw);
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int dw = p.dw, rs = p.dw + 1;
    uint32_t *rows = rows_all + wid * 32 * rs;
    uint32_t *out = rows + lane * rs;
    uint32_t *stage = stage_all[wid];
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = tid; j < p.nb * p.L; j += nthreads) dtab_out[j] = p.etab[j];
    if (tid < pad_floats) dtab_out[p.nb * p.L + tid] = 0.0f;
    const int64_t nwarps = (int64_t)gridDim.x * kDecodeWarps;
    for (int64_t bk0 = ((int64_t)blockIdx.x * kDecodeWarps + wid) * 32; bk0 < p.nb; bk0 += nwarps * 32) {
        const int nrows = (int)min((int64_t)32, p.nb - bk0);
        // the span of stream words the 32 decoders read: from the first bucket's first word to
        // the word after the last bucket's end, plus the two a bit buffer reads ahead
        const uint64_t s0 = p.offs[bk0];
        const uint64_t s1 = bk0 + nrows < p.nb ? p.offs[bk0 + nrows] : p.hdr[0];
        const int64_t w0 = (int64_t)(s0 >> 5);
        const int64_t w1 = min((int64_t)((s1 + 31) >> 5) + 4, p.cap_words);
        const bool staged = w1 - w0 <= kStreamStage;
        if (staged) {
            for (int64_t i = w0 + lane; i < w1; i += 32) stage[i - w0] = __ldg(p.stream + i);
        }
        __syncwarp();
        const int64_t bk = bk0 + lane;
        if (bk < p.nb) {
            const int n = bucket_valid(p, bk);
            const uint64_t start = p.offs[bk];
            if (staged) {
                decode_bucket<B>(dec, decw, start, n, dw, out,
                                 [&](int64_t q) { return q < w1 ? stage[q - w0] : 0u; });
            } else {
                decode_bucket<B>(dec, decw, start, n, dw, out, [&](int64_t q) { return stream_word(p, q); });
            }
        }
        __syncwarp();
        uint32_t *dst = dense_out + bk0 * dw;
        for (int r = 0; r < nrows; ++r)
            for (int j = lane; j < dw; j += 32) dst[r * dw + j] = rows[r * rs + j];
        __syncwarp();
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
    // group encoding table: G codes of one index, their codewords one after the other
    const int G = l.b == 3 ? 2 : 8 / l.b;
    for (int idx = 0; idx < 256; ++idx) {
        uint32_t bitsv = 0;
        int len = 0;
        if (idx < (1 << (G * l.b))) {
            for (int k = 0; k < G; ++k) {
                const int c = (idx >> (l.b * k)) & ((1 << l.b) - 1);
                const uint32_t cw = (uint32_t)(((c < 8 ? p.cw_lo : p.cw_hi) >> (8 * (c & 7))) & 0xFFu);
                bitsv |= cw << len;
                len += (int)((p.len_tab >> (4 * c)) & 15u);
            }
        }
        p.enc[idx] = bitsv | ((uint32_t)len << 24);
    }
    return p;
}

// Grid of a thread-per-bucket kernel (warps of 32 buckets, kBktWarps per CTA): the resident CTAs
// or fewer; -1 if the shared memory cannot be granted.
int bucket_grid(const void *kern, int64_t nb, size_t smem)
{
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return -1;
    int dev = 0, sms = 148, per_sm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBktWarps * 32, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t want = (nb + 32 * kBktWarps - 1) / (32 * kBktWarps);
    return (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * per_sm));
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
    auto count = l.b == 2 ? k_count<2> : l.b == 3 ? k_count<3> : k_count<4>;
    auto encode = l.b == 2 ? k_encode<2> : l.b == 3 ? k_encode<3> : k_encode<4>;
    const size_t smem = sizeof(uint32_t) * kBktWarps * 32 * (size_t)(p.dw + 1);
    const int gc = bucket_grid(reinterpret_cast<const void *>(count), l.nb, smem);
    const int ge = bucket_grid(reinterpret_cast<const void *>(encode), l.nb, smem);
    if (gc < 0 || ge < 0) return GQ_ERR_CUDA;
    count<<<gc, kBktWarps * 32, smem, s>>>(p);
    k_tile_sums<<<(unsigned)p.ntiles, kScanThreads, 0, s>>>(p);
    k_scan_top<<<1, kScanThreads, 0, s>>>(p);
    k_scan_apply<<<(unsigned)p.ntiles, kScanThreads, 0, s>>>(p);
    const int64_t tab = l.nb * l.L;
    encode<<<ge, kBktWarps * 32, smem, s>>>(p, (int)(((tab + 3) & ~int64_t(3)) - tab));
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
    auto decode = l.b == 2 ? k_decode<2> : l.b == 3 ? k_decode<3> : k_decode<4>;
    const size_t smem = sizeof(uint32_t) * kDecodeWarps * 32 * (size_t)(p.dw + 1);
    if (cudaFuncSetAttribute(decode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GQ_ERR_CUDA;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode, kDecodeWarps * 32, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t want = (l.nb + 32 * kDecodeWarps - 1) / (32 * kDecodeWarps);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * per_sm));
    decode<<<(unsigned)grid, kDecodeWarps * 32, smem, static_cast<cudaStream_t>(stream)>>>(
        p, reinterpret_cast<float *>(m + l.dense_levels_off), reinterpret_cast<uint32_t *>(m), pad);
    return cudaGetLastError() == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}

}  // extern "C"
