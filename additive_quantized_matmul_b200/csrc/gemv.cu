// Decode-time product y = diag(s) W x for batch 1..16 on CUDA cores (sm_100a).
//
// W is never materialised: each 8-weight group is rebuilt from its codes on
// the fly (AQLM wiki entry, "Niveau intermédiaire": w ~ sum_k C_k[i_k];
// devtrends.ru summary, "Как это работает технически?": groups of 8) and
// multiplied with the matching 8 activations; the products the paper's
// abstract names for token generation.
//
// Work decomposition shared by the kernels: a warp owns one 8-row tile and
// a set of 32-group blocks; lane l takes group 32*gb + l and loads the
// 16-byte packed chunk holding that group's code word for all 8 rows, so
// one warp load streams 512 contiguous bytes of codes.  Each lane keeps
// eight row accumulators; a 9-shuffle reduce-scatter sums them over lanes.
// Split-K partial sums go to the workspace and the last CTA to arrive for a
// row range adds them in a fixed order (no float atomics: results are
// bit-reproducible).
#include "aq_common.cuh"

namespace aqk {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

struct SplitK {
    float *partials;      // [ks][rows8][batch]
    unsigned *counters;   // [grid.x]
};

// Called by every thread of a CTA after it stored its partial sums for rows
// [row0, row0 + nrows), columns [col0, col0 + ncols) of split blockIdx.y.
// The last CTA of the row range to arrive reduces the splits in split order
// and writes y.
__device__ __forceinline__ void splitk_finish(const Geom &L, SplitK sk, int row0, int nrows,
                                              int batch, int col0, int ncols,
                                              const uint16_t *__restrict__ scales,
                                              uint16_t *__restrict__ y)
{
    __shared__ unsigned s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev = atomicAdd(&sk.counters[blockIdx.x], 1u);
        s_last = (prev == gridDim.y - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int ks = gridDim.y;
    const size_t stride = (size_t)L.rows8 * batch;
    for (int e = threadIdx.x; e < nrows * ncols; e += blockDim.x) {
        int row = row0 + e / ncols;
        int b = col0 + e % ncols;
        if (row >= L.out) continue;
        const float *p = sk.partials + (size_t)row * batch + b;
        float v = 0.f;
        for (int s = 0; s < ks; ++s) v += __ldcg(p + s * stride);
        float sc = scales ? __half2float(__ushort_as_half(scales[row])) : 1.f;
        y[(size_t)row * batch + b] = __half_as_ushort(__float2half_rn(sc * v));
    }
    if (threadIdx.x == 0) sk.counters[blockIdx.x] = 0u;  // ready for the next call
}

// ---------------------------------------------------------------------------
// Row-warp kernel: any scheme, NB batch columns per pass (NB in {1, 2, 4}).
// grid = (row tiles, splits); block = 8 warps, warp w of split s takes group
// blocks gb0 + w, gb0 + w + 8, ... of the split's range.
// ---------------------------------------------------------------------------
template <int K, int NB>
__global__ void __launch_bounds__(kThreads)
gemv_rowwarp_kernel(Geom L, const uint4 *__restrict__ packed, const uint4 *__restrict__ cb,
                    const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x,
                    int batch, int col0, uint16_t *__restrict__ y, SplitK sk, int gbs_per_split)
{
    __shared__ uint4 scb[K == 2 ? 512 : 1];
    __shared__ float red[kWarps][8][NB];
    if (K == 2) {
        for (int i = threadIdx.x; i < 512; i += kThreads) scb[i] = cb[i];
        __syncthreads();
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rt = blockIdx.x;
    const int gb0 = blockIdx.y * gbs_per_split;
    const int gb1 = min(L.gblocks, gb0 + gbs_per_split);
    const int ncols = min(NB, batch - col0);

    float acc[8][NB];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;

    for (int gb = gb0 + warp; gb < gb1; gb += kWarps) {
        const int g = gb * 32 + lane;
        if (g >= L.G) continue;  // padded group: no activations
        const uint4 chunk = ldg_stream_v4(packed + (size_t)rt * L.gp + g);
        uint4 xg[NB];
        if (NB == 1 && batch == 1) {
            xg[0] = ldg_nc_v4(x + (size_t)g * 8);
        } else {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                uint16_t h[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    h[j] = (b < ncols) ? x[((size_t)g * 8 + j) * batch + col0 + b] : (uint16_t)0;
                xg[b] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16),
                                   h[4] | (h[5] << 16), h[6] | (h[7] << 16));
            }
        }
        const uint32_t wd[8] = {chunk.x & 0xffff, chunk.x >> 16, chunk.y & 0xffff, chunk.y >> 16,
                                chunk.z & 0xffff, chunk.z >> 16, chunk.w & 0xffff, chunk.w >> 16};
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            uint4 wv;
            if (K == 1)
                wv = ldg_nc_v4(cb + wd[r]);
            else
                wv = add_round_h8(scb[wd[r] & 0xff], scb[256 + (wd[r] >> 8)]);
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[r][b] = dot8(wv, xg[b], acc[r][b]);
        }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        float col[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) col[r] = acc[r][b];
        float v = warp_reduce8(col, lane);
        if ((lane & 3) == 0) red[warp][reduced_row_of_lane(lane)][b] = v;
    }
    __syncthreads();
    // Fixed-order sum over warps: thread t < 8*ncols owns (row, column).
    const int row0 = rt * 8;
    if (gridDim.y == 1) {
        if (threadIdx.x < 8 * NB) {
            int r = threadIdx.x / NB, b = threadIdx.x % NB;
            int row = row0 + r;
            if (b < ncols && row < L.out) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v += red[w][r][b];
                float sc = scales ? __half2float(__ushort_as_half(scales[row])) : 1.f;
                y[(size_t)row * batch + col0 + b] = __half_as_ushort(__float2half_rn(sc * v));
            }
        }
        return;
    }
    if (threadIdx.x < 8 * NB) {
        int r = threadIdx.x / NB, b = threadIdx.x % NB;
        if (b < ncols) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += red[w][r][b];
            sk.partials[(size_t)blockIdx.y * L.rows8 * batch + (size_t)(row0 + r) * batch + col0 + b] = v;
        }
    }
    // Column chunks of a batch > 4 are separate stream-ordered launches; the
    // last CTA of each resets the counter before the next launch starts.
    splitk_finish(L, sk, row0, 8, batch, col0, ncols, scales, y);
}

// ---------------------------------------------------------------------------
// 2x8, batch 1: per-group codebook x activation lookup tables.
//
// For one block of 32 groups the CTA tabulates L_k[g][c] = <C_k[c], x_g> for
// both codebooks (2 x 256 x 32 fp32 = 64 KiB of shared memory), laid out
// lane-private: entry (k, c, lane) at word (k*256 + c)*32 + lane, so lane l
// (group 32*gb + l) always reads bank l and random codes never conflict.
// A row's contribution from the block is then two table reads per group.
// grid = (row ranges, group blocks); each CTA is one split of the K sum.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
gemv_2x8_lut_kernel(Geom L, const uint4 *__restrict__ packed, const uint4 *__restrict__ cb,
                    const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x,
                    uint16_t *__restrict__ y, SplitK sk, int rt_per_cta)
{
    extern __shared__ float lut[];  // [2][256][32]
    __shared__ uint4 xs[32];        // activations of the block's 32 groups
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gb = blockIdx.y;
    if (threadIdx.x < 32) {
        int g = gb * 32 + threadIdx.x;
        xs[threadIdx.x] = (g < L.G) ? ldg_nc_v4(x + (size_t)g * 8) : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 2 * 256 * 32; e += kThreads) {
        const int l = e & 31;
        const int kc = e >> 5;  // k*256 + c
        lut[e] = dot8(ldg_nc_v4(cb + kc), xs[l], 0.f);
    }
    __syncthreads();
    const int rt0 = blockIdx.x * rt_per_cta;
    const int rt1 = min(L.rtiles, rt0 + rt_per_cta);
    const float *lut0 = lut + lane;
    const float *lut1 = lut + 256 * 32 + lane;
    float *part = sk.partials + (size_t)gb * L.rows8;
    for (int rt = rt0 + warp; rt < rt1; rt += kWarps) {
        const uint4 chunk = ldg_stream_v4(packed + (size_t)rt * L.gp + gb * 32 + lane);
        const uint32_t v[4] = {chunk.x, chunk.y, chunk.z, chunk.w};
        float acc[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] = lut0[(v[i] & 0xff) * 32] + lut1[((v[i] >> 8) & 0xff) * 32];
            acc[2 * i + 1] = lut0[((v[i] >> 16) & 0xff) * 32] + lut1[(v[i] >> 24) * 32];
        }
        float r = warp_reduce8(acc, lane);
        if ((lane & 3) == 0) {
            int row = rt * 8 + reduced_row_of_lane(lane);
            if (gridDim.y == 1) {
                if (row < L.out) {
                    float sc = scales ? __half2float(__ushort_as_half(scales[row])) : 1.f;
                    y[row] = __half_as_ushort(__float2half_rn(sc * r));
                }
            } else {
                part[row] = r;
            }
        }
    }
    if (gridDim.y == 1) return;
    splitk_finish(L, sk, rt0 * 8, (rt1 - rt0) * 8, 1, 0, 1, scales, y);
}

}  // namespace aqk

namespace aqh {
using namespace aqk;

namespace {

enum Path { kRowWarp = 0, kLut2x8 = 1 };

struct GemvPlan {
    Path path;
    int ks;             // splits of the group sum (grid.y)
    int gbs_per_split;  // group blocks per split (row-warp path)
    int rt_per_cta;     // row tiles per CTA
    int grid_x;
    size_t ws_bytes;
};

inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }

// Depends on the shape and batch only, so the workspace size can be
// computed on a host without a GPU.
GemvPlan plan_gemv(const Geom &g, int batch)
{
    GemvPlan p{};
    if (batch == 1 && g.K == 2) {
        p.path = kLut2x8;
        p.ks = g.gblocks;
        // enough rows per CTA to amortise the 16K-entry table, ~300 CTAs
        long pairs = (long)g.rtiles * g.gblocks;
        int rt = (int)((pairs + 299) / 300);
        rt = max(rt, 8);
        rt = min(rt, g.rtiles);
        p.rt_per_cta = rt;
        p.grid_x = (g.rtiles + rt - 1) / rt;
        p.gbs_per_split = 1;
    } else {
        p.path = kRowWarp;
        p.rt_per_cta = 1;
        p.grid_x = g.rtiles;
        int ks = (512 + g.rtiles - 1) / g.rtiles;
        ks = max(1, min(ks, min(8, g.gblocks)));
        p.gbs_per_split = (g.gblocks + ks - 1) / ks;
        p.ks = (g.gblocks + p.gbs_per_split - 1) / p.gbs_per_split;
    }
    p.ws_bytes = kWsHeader + align16(sizeof(unsigned) * (size_t)p.grid_x);
    if (p.ks > 1) p.ws_bytes += (size_t)p.ks * g.rows8 * batch * sizeof(float);
    return p;
}

}  // namespace

size_t gemv_workspace_bytes(const Geom &g, int batch) { return plan_gemv(g, batch).ws_bytes; }

cudaError_t launch_gemv(const Geom &g, const void *packed, const uint16_t *cb,
                        const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                        void *ws, cudaStream_t s)
{
    const GemvPlan p = plan_gemv(g, batch);
    SplitK sk;
    char *base = reinterpret_cast<char *>(ws);
    sk.counters = reinterpret_cast<unsigned *>(base + kWsHeader);
    sk.partials = reinterpret_cast<float *>(base + kWsHeader +
                                            align16(sizeof(unsigned) * (size_t)p.grid_x));
    const uint4 *pk = reinterpret_cast<const uint4 *>(packed);
    const uint4 *c = reinterpret_cast<const uint4 *>(cb);
    dim3 grid(p.grid_x, p.ks);
    if (p.path == kLut2x8) {
        const int smem = 2 * 256 * 32 * sizeof(float);
        static bool attr_set = false;  // idempotent, benign race
        if (!attr_set) {
            cudaError_t e = cudaFuncSetAttribute(gemv_2x8_lut_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            attr_set = true;
        }
        gemv_2x8_lut_kernel<<<grid, kThreads, smem, s>>>(g, pk, c, scales, x, y, sk, p.rt_per_cta);
        return cudaGetLastError();
    }
    if (batch == 1) {
        if (g.K == 1)
            gemv_rowwarp_kernel<1, 1><<<grid, kThreads, 0, s>>>(g, pk, c, scales, x, 1, 0, y, sk, p.gbs_per_split);
        else
            gemv_rowwarp_kernel<2, 1><<<grid, kThreads, 0, s>>>(g, pk, c, scales, x, 1, 0, y, sk, p.gbs_per_split);
        return cudaGetLastError();
    }
    const int nb = batch == 2 ? 2 : 4;
    for (int col0 = 0; col0 < batch; col0 += nb) {
        if (g.K == 1) {
            if (nb == 2)
                gemv_rowwarp_kernel<1, 2><<<grid, kThreads, 0, s>>>(g, pk, c, scales, x, batch, col0, y, sk, p.gbs_per_split);
            else
                gemv_rowwarp_kernel<1, 4><<<grid, kThreads, 0, s>>>(g, pk, c, scales, x, batch, col0, y, sk, p.gbs_per_split);
        } else {
            if (nb == 2)
                gemv_rowwarp_kernel<2, 2><<<grid, kThreads, 0, s>>>(g, pk, c, scales, x, batch, col0, y, sk, p.gbs_per_split);
            else
                gemv_rowwarp_kernel<2, 4><<<grid, kThreads, 0, s>>>(g, pk, c, scales, x, batch, col0, y, sk, p.gbs_per_split);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace aqh
