// Code packing, unpacking and dequantisation kernels (sm_100a).
//
// Dequantisation follows the additive decode of "Extreme Compression of
// Large Language Models via Additive Quantization" (AQLM wiki entry, section
// "Niveau intermédiaire": a group of weights is the sum of one codeword from
// each of K codebooks; devtrends.ru summary, "Как это работает технически?":
// groups of 8 consecutive weights): W[o][8g+j] = RN16(sum_k C_k[i_k][j]).
#include "aq_common.cuh"

namespace aqk {

// Word of group g for row o from codes[out][G][K] (u16 for 1x16, u8 pairs for 2x8).
__device__ __forceinline__ uint32_t load_word(const Geom &L, const void *codes, int o, int g)
{
    if (o >= L.out || g >= L.G) return 0u;  // padding
    size_t idx = (size_t)o * L.G + g;
    if (L.K == 1) return reinterpret_cast<const uint16_t *>(codes)[idx];
    const uint8_t *c = reinterpret_cast<const uint8_t *>(codes) + idx * 2;
    return (uint32_t)c[0] | ((uint32_t)c[1] << 8);
}

// One thread per 16-byte chunk (rt, g): 8 rows' words for one group.
__global__ void pack_kernel(Geom L, const void *__restrict__ codes, uint4 *__restrict__ packed)
{
    size_t chunk = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    size_t nchunks = (size_t)L.rtiles * L.gp;
    if (chunk >= nchunks) return;
    int rt = (int)(chunk / L.gp);
    int g = (int)(chunk % L.gp);
    uint32_t w[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) w[r] = load_word(L, codes, rt * 8 + r, g);
    uint4 v;
    v.x = w[0] | (w[1] << 16);
    v.y = w[2] | (w[3] << 16);
    v.z = w[4] | (w[5] << 16);
    v.w = w[6] | (w[7] << 16);
    packed[chunk] = v;
}

__global__ void unpack_kernel(Geom L, const uint4 *__restrict__ packed, void *__restrict__ codes)
{
    size_t chunk = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    size_t nchunks = (size_t)L.rtiles * L.gp;
    if (chunk >= nchunks) return;
    int rt = (int)(chunk / L.gp);
    int g = (int)(chunk % L.gp);
    if (g >= L.G) return;
    uint4 v = packed[chunk];
    uint32_t w[8] = {v.x & 0xffff, v.x >> 16, v.y & 0xffff, v.y >> 16,
                     v.z & 0xffff, v.z >> 16, v.w & 0xffff, v.w >> 16};
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int o = rt * 8 + r;
        if (o >= L.out) break;
        size_t idx = (size_t)o * L.G + g;
        if (L.K == 1) {
            reinterpret_cast<uint16_t *>(codes)[idx] = (uint16_t)w[r];
        } else {
            uint8_t *c = reinterpret_cast<uint8_t *>(codes) + idx * 2;
            c[0] = (uint8_t)(w[r] & 0xff);
            c[1] = (uint8_t)(w[r] >> 8);
        }
    }
}

// Dequantisation: one thread per chunk (rt, g < G).  Lanes of a warp take
// consecutive groups of the same row tile, so each of the 8 row stores is a
// 512-byte contiguous warp write.  2x8 codebooks (8 KiB) are staged in
// shared memory; the 1 MiB 1x16 codebook is read through L2.
template <int K>
__global__ void __launch_bounds__(256) dequant_kernel(Geom L, const uint4 *__restrict__ packed,
                                                      const uint4 *__restrict__ cb,
                                                      const uint16_t *__restrict__ scales,
                                                      uint4 *__restrict__ w)
{
    __shared__ uint4 scb[K == 2 ? 512 : 1];
    if (K == 2) {
        for (int i = threadIdx.x; i < 512; i += blockDim.x) scb[i] = cb[i];
        __syncthreads();
    }
    size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    size_t total = (size_t)L.rtiles * L.G;
    if (t >= total) return;
    int rt = (int)(t / L.G);
    int g = (int)(t % L.G);
    uint4 v = packed[(size_t)rt * L.gp + g];
    uint32_t wd[8] = {v.x & 0xffff, v.x >> 16, v.y & 0xffff, v.y >> 16,
                      v.z & 0xffff, v.z >> 16, v.w & 0xffff, v.w >> 16};
    const size_t row_chunks = (size_t)L.G;  // 16-byte chunks per output row
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int o = rt * 8 + r;
        if (o >= L.out) break;
        uint4 val;
        if (K == 1) {
            val = ldg_nc_v4(cb + wd[r]);  // verbatim codeword, no arithmetic
        } else {
            val = add_round_h8(scb[wd[r] & 0xff], scb[256 + (wd[r] >> 8)]);
        }
        if (scales) {
            float s = __half2float(__ushort_as_half(scales[o]));
            val = scale_round_h8(val, s);
        }
        w[(size_t)o * row_chunks + g] = val;
    }
}

}  // namespace aqk

namespace aqh {
using namespace aqk;

cudaError_t launch_pack(const Geom &g, const void *codes, void *packed, cudaStream_t s)
{
    size_t n = (size_t)g.rtiles * g.gp;
    unsigned blocks = (unsigned)((n + 255) / 256);
    pack_kernel<<<blocks, 256, 0, s>>>(g, codes, reinterpret_cast<uint4 *>(packed));
    return cudaGetLastError();
}

cudaError_t launch_unpack(const Geom &g, const void *packed, void *codes, cudaStream_t s)
{
    size_t n = (size_t)g.rtiles * g.gp;
    unsigned blocks = (unsigned)((n + 255) / 256);
    unpack_kernel<<<blocks, 256, 0, s>>>(g, reinterpret_cast<const uint4 *>(packed), codes);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const Geom &g, const void *packed, const uint16_t *cb,
                           const uint16_t *scales, uint16_t *w, cudaStream_t s)
{
    size_t n = (size_t)g.rtiles * g.G;
    unsigned blocks = (unsigned)((n + 255) / 256);
    const uint4 *p = reinterpret_cast<const uint4 *>(packed);
    const uint4 *c = reinterpret_cast<const uint4 *>(cb);
    uint4 *o = reinterpret_cast<uint4 *>(w);
    if (g.K == 1)
        dequant_kernel<1><<<blocks, 256, 0, s>>>(g, p, c, scales, o);
    else
        dequant_kernel<2><<<blocks, 256, 0, s>>>(g, p, c, scales, o);
    return cudaGetLastError();
}

}  // namespace aqh
