// Quantisation schemes K x B (K codebooks of 2^B codewords, groups of 8
// weights) and the code words of the packed layout.
//
// The schemes are those named by the pages on "Extreme Compression of Large
// Language Models via Additive Quantization": 1x16, 2x8 and 8x8 (devtrends.ru
// summary, "Схемы квантования"), 2x16 (AQLM wiki entry, "Niveau
// intermédiaire", the 4-bit example) and 1x8 (devtrends.ru, notes on 1-bit
// models: 8 bits per group of 8).  Bit rate K*B/8 bits per weight.
//
// Packed word of (row o, group g): W = K*B/8 bytes, code k in bits
// [k*B, (k+1)*B), little-endian.  Chunk (rt, g) = the words of rows
// 8rt..8rt+7 for group g, 8*W contiguous bytes at chunk index rt*Gp + g.
#pragma once

#include "aq_common.cuh"

namespace aqk {

template <int K_, int B_>
struct Scheme {
    static constexpr int K = K_, B = B_;
    static constexpr int kWordBytes = K * B / 8;
    static constexpr int kChunkBytes = 8 * kWordBytes;     // 8, 16, 32 or 64
    static constexpr int kChunkWords = kChunkBytes / 4;    // 32-bit words per chunk
    static constexpr bool kBooksInSmem = (B == 8);         // K x 4 KiB of codebooks
    static constexpr int kSmemBookBytes = kBooksInSmem ? K * 256 * 16 : 0;
    static constexpr bool kVerbatim = (K == 1);            // weight = one codeword, no arithmetic
    static constexpr uint32_t kMask = (1u << B) - 1u;
};

// The schemes the library accepts.
inline bool scheme_supported(int K, int B)
{
    return (K == 1 && B == 16) || (K == 2 && B == 8) || (K == 1 && B == 8) || (K == 2 && B == 16) ||
           (K == 8 && B == 8);
}

// Calls f(Scheme<K, B>{}) for the layer's scheme (checked by the caller).
template <class F>
cudaError_t with_scheme(const Geom &g, F &&f)
{
    if (g.K == 1 && g.B == 16) return f(Scheme<1, 16>{});
    if (g.K == 2 && g.B == 8) return f(Scheme<2, 8>{});
    if (g.K == 1 && g.B == 8) return f(Scheme<1, 8>{});
    if (g.K == 2 && g.B == 16) return f(Scheme<2, 16>{});
    if (g.K == 8 && g.B == 8) return f(Scheme<8, 8>{});
    return cudaErrorInvalidValue;
}

// One chunk held in registers.
template <class S>
struct Chunk {
    uint32_t w[S::kChunkWords];

    // Code k of row r of the chunk (r, k compile-time after unrolling).
    __device__ __forceinline__ uint32_t code(int r, int k) const
    {
        const int bit = r * S::kWordBytes * 8 + k * S::B;
        return (w[bit >> 5] >> (bit & 31)) & S::kMask;
    }
};

// Chunk (rt, g) of the packed codes; zero when `live` is false.  The load
// is issued where it is written (a prefetch), not at its first use.
template <class S>
__device__ __forceinline__ Chunk<S> load_chunk(const uint8_t *__restrict__ packed, size_t chunk_index, bool live)
{
    Chunk<S> c;
    const uint8_t *p = packed + chunk_index * S::kChunkBytes;
    if constexpr (S::kChunkBytes == 8) {
        uint32_t a = 0, b = 0;
        if (live)
            asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "l"(p));
        c.w[0] = a;
        c.w[1] = b;
    } else {
#pragma unroll
        for (int q = 0; q < S::kChunkBytes / 16; ++q) {
            const uint4 v = live ? ldg_stream_v4(p + 16 * q) : make_uint4(0, 0, 0, 0);
            c.w[4 * q + 0] = v.x;
            c.w[4 * q + 1] = v.y;
            c.w[4 * q + 2] = v.z;
            c.w[4 * q + 3] = v.w;
        }
    }
    return c;
}

__device__ __forceinline__ uint32_t u4_at(const uint4 &v, int h)
{
    return h == 0 ? v.x : h == 1 ? v.y : h == 2 ? v.z : v.w;
}

// Sum of K binary16 8-vectors, one rounding to binary16, exact: the terms
// are added in double (at most eight binary16 terms, exactly representable)
// and rounded once.  Used where the decoded weights are the output.
template <int K>
__device__ __forceinline__ uint4 sum_round_exact_h8(const uint4 (&t)[K])
{
    uint32_t out[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        double lo = 0.0, hi = 0.0;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const uint32_t v = u4_at(t[k], h);
            const float2 f = h2f2(v);
            lo = (k == 0) ? (double)f.x : lo + (double)f.x;
            hi = (k == 0) ? (double)f.y : hi + (double)f.y;
        }
        out[h] = (uint32_t)__half_as_ushort(__double2half(lo)) | ((uint32_t)__half_as_ushort(__double2half(hi)) << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// Sum of K binary16 8-vectors accumulated in fp32 and rounded to binary16.
// Used where the decoded weights only feed a product (tolerance-checked):
// for K = 2 the fp32 sum of two binary16 values is exact, so this equals the
// exact decode; for K = 8 it may differ from it by one rounding.
template <int K>
__device__ __forceinline__ uint4 sum_round_fast_h8(const uint4 (&t)[K])
{
    if constexpr (K == 1) {
        return t[0];
    } else if constexpr (K == 2) {
        return add_round_h8(t[0], t[1]);
    } else {
        uint32_t out[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            float2 acc = h2f2(u4_at(t[0], h));
#pragma unroll
            for (int k = 1; k < K; ++k) {
                const float2 f = h2f2(u4_at(t[k], h));
                acc.x += f.x;
                acc.y += f.y;
            }
            out[h] = f2h2(acc.x, acc.y);
        }
        return make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// The K codewords of row r of a chunk: from shared memory (B = 8, books
// laid out [k][256]) or through L2 (B = 16, books [k][65536]).
template <class S>
__device__ __forceinline__ void gather_terms(const Chunk<S> &c, int r, const uint4 *__restrict__ smem_books,
                                             const uint4 *__restrict__ gmem_books, uint4 (&t)[S::K])
{
#pragma unroll
    for (int k = 0; k < S::K; ++k) {
        const uint32_t code = c.code(r, k);
        if constexpr (S::kBooksInSmem)
            t[k] = smem_books[k * 256 + code];
        else
            t[k] = ldg_nc_v4(gmem_books + ((size_t)k << S::B) + code);
    }
}

}  // namespace aqk
