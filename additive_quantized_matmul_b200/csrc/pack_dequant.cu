// Code packing, unpacking and dequantisation kernels (sm_100a).
//
// Dequantisation follows the additive decode of "Extreme Compression of
// Large Language Models via Additive Quantization" (AQLM wiki entry, section
// "Niveau intermédiaire": a group of weights is the sum of one codeword from
// each of K codebooks; devtrends.ru summary, "Как это работает технически?":
// groups of 8 consecutive weights): W[o][8g+j] = RN16(sum_k C_k[i_k][j]).
#include "scheme.cuh"

namespace aqk {

// Code k of group g of row o from codes[out][G][K] (u8 for B = 8, u16 for
// B = 16); zero for padding rows and groups.
template <class S>
__device__ __forceinline__ uint32_t load_code(const Geom &L, const void *codes, int o, int g, int k)
{
    if (o >= L.out || g >= L.G) return 0u;
    const size_t idx = ((size_t)o * L.G + g) * S::K + k;
    if constexpr (S::B <= 8)
        return reinterpret_cast<const uint8_t *>(codes)[idx];
    else
        return reinterpret_cast<const uint16_t *>(codes)[idx];
}

// One thread per chunk (rt, g): the 8 rows' words of one group.
template <class S>
__global__ void pack_kernel(Geom L, const void *__restrict__ codes, uint8_t *__restrict__ packed)
{
    const size_t chunk = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (chunk >= (size_t)L.rtiles * L.gp) return;
    const int rt = (int)(chunk / L.gp), g = (int)(chunk % L.gp);
    Chunk<S> c;
#pragma unroll
    for (int i = 0; i < S::kChunkWords; ++i) c.w[i] = 0u;
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int k = 0; k < S::K; ++k) {
            const int bit = r * S::kWordBytes * 8 + k * S::B;
            c.w[bit >> 5] |= load_code<S>(L, codes, rt * 8 + r, g, k) << (bit & 31);
        }
    uint32_t *dst = reinterpret_cast<uint32_t *>(packed + chunk * S::kChunkBytes);
    if constexpr (S::kChunkBytes == 8) {
        *reinterpret_cast<uint2 *>(dst) = make_uint2(c.w[0], c.w[1]);
    } else {
#pragma unroll
        for (int q = 0; q < S::kChunkBytes / 16; ++q)
            reinterpret_cast<uint4 *>(dst)[q] = make_uint4(c.w[4 * q], c.w[4 * q + 1], c.w[4 * q + 2], c.w[4 * q + 3]);
    }
}

template <class S>
__global__ void unpack_kernel(Geom L, const uint8_t *__restrict__ packed, void *__restrict__ codes)
{
    const size_t chunk = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (chunk >= (size_t)L.rtiles * L.gp) return;
    const int rt = (int)(chunk / L.gp), g = (int)(chunk % L.gp);
    if (g >= L.G) return;
    const Chunk<S> c = load_chunk<S>(packed, chunk, true);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int o = rt * 8 + r;
        if (o >= L.out) break;
#pragma unroll
        for (int k = 0; k < S::K; ++k) {
            const size_t idx = ((size_t)o * L.G + g) * S::K + k;
            if constexpr (S::B <= 8)
                reinterpret_cast<uint8_t *>(codes)[idx] = (uint8_t)c.code(r, k);
            else
                reinterpret_cast<uint16_t *>(codes)[idx] = (uint16_t)c.code(r, k);
        }
    }
}

// Dequantisation: one thread per chunk (rt, g < G).  Lanes of a warp take
// consecutive groups of the same row tile, so each of the 8 row stores is a
// 512-byte contiguous warp write.  B = 8 codebooks (K x 4 KiB) are staged in
// shared memory; B = 16 codebooks (1 MiB each) are read through L2.  The
// K-term sum is exact and rounded once.
template <class S>
__global__ void __launch_bounds__(256) dequant_kernel(Geom L, const uint8_t *__restrict__ packed,
                                                      const uint4 *__restrict__ cb,
                                                      const uint16_t *__restrict__ scales,
                                                      uint4 *__restrict__ w)
{
    __shared__ uint4 scb[S::kBooksInSmem ? S::K * 256 : 1];
    if constexpr (S::kBooksInSmem) {
        for (int i = threadIdx.x; i < S::K * 256; i += blockDim.x) scb[i] = cb[i];
        __syncthreads();
    }
    const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (size_t)L.rtiles * L.G) return;
    const int rt = (int)(t / L.G), g = (int)(t % L.G);
    const Chunk<S> c = load_chunk<S>(packed, (size_t)rt * L.gp + g, true);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int o = rt * 8 + r;
        if (o >= L.out) break;
        uint4 terms[S::K];
        gather_terms<S>(c, r, scb, cb, terms);
        uint4 val;
        if constexpr (S::K <= 2)
            val = sum_round_fast_h8<S::K>(terms);  // exact for one or two terms
        else
            val = sum_round_exact_h8<S::K>(terms);
        if (scales) val = scale_round_h8(val, __half2float(__ushort_as_half(scales[o])));
        w[(size_t)o * L.G + g] = val;
    }
}

}  // namespace aqk

namespace aqh {
using namespace aqk;

cudaError_t launch_pack(const Geom &g, const void *codes, void *packed, cudaStream_t s)
{
    const size_t n = (size_t)g.rtiles * g.gp;
    const unsigned blocks = (unsigned)((n + 255) / 256);
    return with_scheme(g, [&](auto sch) {
        pack_kernel<decltype(sch)><<<blocks, 256, 0, s>>>(g, codes, reinterpret_cast<uint8_t *>(packed));
        return cudaGetLastError();
    });
}

cudaError_t launch_unpack(const Geom &g, const void *packed, void *codes, cudaStream_t s)
{
    const size_t n = (size_t)g.rtiles * g.gp;
    const unsigned blocks = (unsigned)((n + 255) / 256);
    return with_scheme(g, [&](auto sch) {
        unpack_kernel<decltype(sch)><<<blocks, 256, 0, s>>>(g, reinterpret_cast<const uint8_t *>(packed), codes);
        return cudaGetLastError();
    });
}

cudaError_t launch_dequant(const Geom &g, const void *packed, const uint16_t *cb,
                           const uint16_t *scales, uint16_t *w, cudaStream_t s)
{
    const size_t n = (size_t)g.rtiles * g.G;
    const unsigned blocks = (unsigned)((n + 255) / 256);
    return with_scheme(g, [&](auto sch) {
        dequant_kernel<decltype(sch)><<<blocks, 256, 0, s>>>(g, reinterpret_cast<const uint8_t *>(packed),
                                                             reinterpret_cast<const uint4 *>(cb), scales,
                                                             reinterpret_cast<uint4 *>(w));
        return cudaGetLastError();
    });
}

}  // namespace aqh
