// Decode-time product y = diag(s) W x for batch 1..16 (sm_100a).
//
// W is never materialised in HBM: each 8-weight group is rebuilt from its
// codes on the fly (AQLM wiki entry, "Niveau intermédiaire": w ~ sum_k
// C_k[i_k]; devtrends.ru summary, "Как это работает технически?": groups of
// 8) and multiplied with the matching 8 activations, the product the
// paper's abstract names for token generation.
//
// Three kernels, chosen by scheme, batch and shape:
//  * 8-bit codes with one or two codebooks (1x8, 2x8), batch 1 --
//    `gemv_lut_kernel`: per-group codebook x activation tables in shared
//    memory, lane-private so random codes never conflict; K 4-byte table
//    reads per group.
//  * 1x16 at batch 1 and 2 (unless the layer has too few rows to fill the
//    SMs without more than 32 splits per row range) -- `gemv_1x16_cc_kernel`:
//    codewords read into registers through L1 and multiplied with x on the
//    CUDA cores, no tile in shared memory.
//  * every other case -- `gemv_tc_kernel`: codes are decoded into a 128x64
//    binary16 tile in shared memory (128-byte-swizzled, K-major) and
//    multiplied by the activations on the tensor cores (tcgen05.mma,
//    M = 128, N = 16, fp32 accumulator in tensor memory), so the cost per
//    group does not grow with the batch.
// For 1x16 the bound is the rate of random 16-byte codeword reads from the
// 1 MiB codebook (through L2, partly L1), not HBM.
// Split-K partial sums go to the workspace and the last CTA to arrive for a
// row range adds them in split order (no float atomics: bit-reproducible).
#include <algorithm>
#include <mutex>
#include <type_traits>

#include <cuda.h>  // driver types only; the calls are fetched at run time

#include "scheme.cuh"
#include "tc_common.cuh"

namespace aqk {

struct SplitK {
    float *partials;      // [slots][rows8][batch]
    unsigned *counters;   // one per row range
};

// Scales the float4 of outputs starting at element idx of a row block
// ([rows][batch], rows from row0), rounds once to binary16 and stores it.
// s_sc: the block's scales in shared memory (or null: read them here).
// Batch a multiple of 4: one row, one 8-byte store; batch 1: four rows,
// one 8-byte scale read and one 8-byte store.
__device__ __forceinline__ void finish_store4(const Geom &L, int row0, int idx, int batch, float4 acc,
                                              const uint16_t *__restrict__ scales, const float *s_sc,
                                              uint16_t *__restrict__ y)
{
    if ((batch & 3) == 0) {
        const int r = idx / batch, row = row0 + r;
        if (row >= L.out) return;
        const float sc = s_sc ? s_sc[r] : (scales ? __half2float(__ushort_as_half(scales[row])) : 1.f);
        *reinterpret_cast<uint2 *>(y + (size_t)row * batch + idx % batch) =
            make_uint2(f2h2(sc * acc.x, sc * acc.y), f2h2(sc * acc.z, sc * acc.w));
        return;
    }
    const float v[4] = {acc.x, acc.y, acc.z, acc.w};
    if (batch == 1 && row0 + idx + 3 < L.out) {
        float sc[4] = {1.f, 1.f, 1.f, 1.f};
        if (s_sc) {
#pragma unroll
            for (int c = 0; c < 4; ++c) sc[c] = s_sc[idx + c];
        } else if (scales) {
            const uint2 w = *reinterpret_cast<const uint2 *>(scales + row0 + idx);  // row0 + idx: a multiple of 4
            const float2 lo = h2f2(w.x), hi = h2f2(w.y);
            sc[0] = lo.x, sc[1] = lo.y, sc[2] = hi.x, sc[3] = hi.y;
        }
        *reinterpret_cast<uint2 *>(y + row0 + idx) =
            make_uint2(f2h2(sc[0] * v[0], sc[1] * v[1]), f2h2(sc[2] * v[2], sc[3] * v[3]));
        return;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int r = (idx + c) / batch, row = row0 + r;
        if (row < L.out) {
            const float sc = s_sc ? s_sc[r] : (scales ? __half2float(__ushort_as_half(scales[row])) : 1.f);
            y[(size_t)row * batch + (idx + c) % batch] = __half_as_ushort(__float2half_rn(sc * v[c]));
        }
    }
}

// Rows whose scales the split-K finish keeps in shared memory.
constexpr int kFinishScaleRows = 256;

// The split-K finish of rows [row0, row0 + nrows) reads their scales at the
// end of the launch; one CTA of the row range brings them into L2 at its
// start (a prefetch returns nothing, so it may precede the dependency wait).
__device__ __forceinline__ void prefetch_range_scales(const Geom &L, const uint16_t *scales, int row0, int nrows)
{
    if (threadIdx.x != 0 || blockIdx.y != 0 || gridDim.y == 1 || !scales) return;
    const int n = (min(row0 + nrows, L.out) - row0) & ~7;  // whole 16-byte pieces inside the array
    if (n > 0) prefetch_l2_bulk(scales + row0, (uint32_t)n * 2u);
}

// Called by every thread of a CTA after it stored its partial sums for rows
// [row0, row0 + nrows), columns [0, batch), into its slot of that row range
// (nrows is a multiple of 8 and row0 + nrows <= rows8, so the block is a
// whole number of float4 inside every slot).  The row range has `ks` slots
// and arrival counter `counter`; the last CTA to arrive reduces the slots in
// slot order, writes y and resets the counter for the next call.  With
// `stage` (shared memory the CTA no longer needs, `stage_bytes` of it, 16-byte
// aligned) the partial sums are staged there: a pass takes the same float4
// range of every slot, one contiguous run per slot, by one bulk copy each
// (TMA engine), and the range's scales are read into shared memory
// meanwhile.
// Without it (or with fewer than 16 ks bytes) they are summed straight
// from L2, eight slots in flight per float4.
template <int kInFlight = 8>
__device__ __forceinline__ void splitk_finish(const Geom &L, SplitK sk, int counter, int ks, int row0,
                                              int nrows, int batch, const uint16_t *__restrict__ scales,
                                              uint16_t *__restrict__ y, float4 *stage, int stage_bytes)
{
    __shared__ unsigned s_last;
    __shared__ float s_scale[kFinishScaleRows];
    __shared__ uint64_t s_staged;  // the bulk copies of a pass have landed
    __syncthreads();
    if (threadIdx.x == 0) {
        // the barrier orders the CTA's partial stores before this thread's
        // increment, whose release publishes them; its acquire orders the
        // last CTA's reads after every slot's
        const unsigned prev = atom_add_acq_rel_gpu(&sk.counters[counter], 1u);
        s_last = (prev == (unsigned)ks - 1u) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_last) return;
    const size_t vstride = (size_t)L.rows8 * batch / 4;
    const float4 *base = reinterpret_cast<const float4 *>(sk.partials + (size_t)row0 * batch);
    const int nvec = nrows * batch / 4;
    const int chunk = min(nvec, stage_bytes / (16 * ks));  // float4 elements per pass
    if (chunk == 0) {
        // no staging area, or more slots than it holds
        for (int e = threadIdx.x; e < nvec; e += blockDim.x) {
            float4 acc = __ldcg(base + e);
            for (int s0 = 1; s0 < ks; s0 += kInFlight) {
                float4 t[kInFlight];
#pragma unroll
                for (int j = 0; j < kInFlight; ++j)
                    if (s0 + j < ks) t[j] = __ldcg(base + (size_t)(s0 + j) * vstride + e);
#pragma unroll
                for (int j = 0; j < kInFlight; ++j)
                    if (s0 + j < ks) {
                        acc.x += t[j].x; acc.y += t[j].y; acc.z += t[j].z; acc.w += t[j].w;
                    }
            }
            finish_store4(L, row0, e * 4, batch, acc, scales, nullptr, y);
        }
    }
    const bool pre = scales && nrows <= kFinishScaleRows;  // scales staged too
    for (int c0 = 0, pass = 0; chunk > 0 && c0 < nvec; c0 += chunk, ++pass) {
        const int n = min(chunk, nvec - c0);
        if (threadIdx.x == 0) {
            if (pass == 0) {
                mbar_init(&s_staged, 1);
                fence_mbar_init();
            }
            fence_proxy_async_global();  // the slots' stores, acquired above, before the bulk reads
            fence_proxy_async_smem();    // the CTA's earlier use of the staging area before the bulk writes
            mbar_arrive_expect_tx(&s_staged, (uint32_t)(ks * n * 16));
            for (int sl = 0; sl < ks; ++sl)
                bulk_load(smem_u32(stage + (size_t)sl * n), base + (size_t)sl * vstride + c0, (uint32_t)(n * 16),
                          &s_staged);
        }
        if (pre && c0 == 0)  // while the copies are in flight
            for (int i = threadIdx.x; i < nrows; i += blockDim.x)
                s_scale[i] = row0 + i < L.out ? __half2float(__ushort_as_half(scales[row0 + i])) : 0.f;
        __syncthreads();  // the barrier's initialisation and the scales
        if (!mbar_wait_ns(&s_staged, pass & 1, kWaitNs) && threadIdx.x == 0)
            record_status(reinterpret_cast<char *>(sk.counters) - kWsHeader, AQ_ERR_TIMEOUT);
        for (int e = threadIdx.x; e < n; e += blockDim.x) {
            float4 acc = stage[e];
            for (int sl = 1; sl < ks; ++sl) {
                const float4 t = stage[sl * n + e];
                acc.x += t.x; acc.y += t.y; acc.z += t.z; acc.w += t.w;
            }
            finish_store4(L, row0, (c0 + e) * 4, batch, acc, scales, pre ? s_scale : nullptr, y);
        }
        __syncthreads();  // the next pass reuses the staging area
    }
    if (threadIdx.x == 0) sk.counters[counter] = 0u;
}

// ---------------------------------------------------------------------------
// 8-bit codes with one or two codebooks (2x8, 1x8), batch 1: per-group
// codebook x activation tables in binary16.
//
// A CTA covers a range of 8-row tiles and kLutGroups(K) groups: 64 for
// 2x8, 128 for 1x8.  For those groups it tabulates L_k[g][c] = <C_k[c], x_g>
// (each product of two binary16 values is exact in fp32; the 8-term sum is
// rounded once to fp32, then once to binary16) in 64 KiB of shared memory:
// word (c, q, l) at c*64 + q*32 + l holds the entries of local groups
// g0 + l (low half) and g0 + 32 + l (high half), where q is the codebook
// (2x8, g0 = 0) or the half of the group range (1x8, g0 = 64 q).  Lane l
// handles exactly the groups whose entries sit in bank l, so random codes
// never conflict; a lookup's byte offset c*256 + l*4 is one byte permute of
// the code byte and l*4, and q*128 + half*2 go into the load's immediate.
// Each row and lane takes four lookups (two groups x two codebooks, or four
// groups), summed in binary16, and a warp reduction adds the lanes in fp32.
//
// The tables are one small matrix product T = X C^T (groups x codewords,
// inner size 8) on mma.sync m16n8k8, binary16 operands, fp32 accumulators:
// groups on M, codewords on N, so a lane's fragment holds groups gid, gid+8
// of two tiles 32 groups apart (one word each); lanes rotate their four
// word slots by their index within the quad so that every store covers 32
// distinct banks.  Binary16 entries need |L| < 65504: the CTA bounds them
// by 8 max|x| max|C| over its groups and codebooks, and when the bound
// fails (or an input is not finite) it skips the tables and decodes each
// weight group exactly (sum of the codewords rounded once, as the
// dequantised matrix has it) and multiplies it in fp32 instead.
//
// 16 warps; warp w takes the CTA's row tiles w, w + 16, ...  A tile's codes
// for the CTA's groups are one contiguous kilobyte of the packed layout;
// each warp copies its tiles into a ring of its own in shared memory with
// cp.async, kLutRing tiles ahead.  The codebooks, the first tiles of codes
// and an L2 prefetch of the rest are requested before the CTA waits for the
// previous launch.  grid = (row ranges, group splits), about one CTA per
// SM, small enough (registers, shared memory) for a CTA of the next launch
// to start beside it; each CTA is one split of the sum, finished by the
// last CTA of the row range.
// ---------------------------------------------------------------------------
constexpr int kLutWarps = 16;
constexpr int kLutThreads = kLutWarps * 32;
constexpr int kLutBytes = 256 * 64 * 4;  // the tables: 256 codes x 64 words
constexpr int kLutRing = 2;              // row tiles of codes in flight per warp
constexpr int kLutTileBytes = 1024;      // codes of one row tile for the CTA's groups
constexpr int kLutSmem = kLutBytes + kLutWarps * kLutRing * kLutTileBytes;  // dynamic shared memory
template <int K>
constexpr int kLutGroups = 128 / K;      // groups per CTA: 64 (2x8) or 128 (1x8)

// D = A(16x8, row) * B(8x8, col), binary16 in, fp32 out (no addend).
__device__ __forceinline__ void mma_m16n8k8(float d[4], uint32_t a0, uint32_t a1, uint32_t b0)
{
    asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0), "f"(0.f));
}

// Byte offset c*256 + lane4 of the table row of code (r, k) of a chunk
// (8-bit codes: code (r, k) is byte r*K + k of the chunk) by one byte
// permute: the code byte goes to byte 1, lane4 (< 256) to byte 0.
template <class S>
__device__ __forceinline__ uint32_t lut_offset(const Chunk<S> &c, int r, int k, uint32_t lane4)
{
    const int bi = r * S::K + k;
    const uint32_t sel = 0x5504u | ((uint32_t)(bi & 3) << 4);
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(c.w[bi >> 2]), "r"(lane4), "r"(sel));
    return d;
}

// Largest |v| over eight binary16 values, as the bits of a non-negative
// binary16 (NaN orders above infinity).
__device__ __forceinline__ uint32_t absmax_h8_bits(uint4 v)
{
    uint32_t m = 0;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7fffu, (w[i] >> 16) & 0x7fffu));
    return m;
}

// The table path's fallback: each row's weight groups decoded exactly
// (codewords from the codebooks in shared memory, summed with one binary16
// rounding) and multiplied with the activations in fp32.
// kStaged: the split-K finish stages the slots in shared memory (chosen
// for more than 8 slots: Llama-2-7B 4096x11008, 22 slots, 10.7 -> 9.8 us;
// 11008x4096, 8 slots, 8.5 -> 8.7 us when staged).
template <class S, bool kStaged>
__global__ void __launch_bounds__(kLutThreads, 2)
gemv_lut_kernel(Geom L, const uint8_t *__restrict__ packed, const uint4 *__restrict__ cb,
                const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x,
                uint16_t *__restrict__ y, SplitK sk, int rt_per_cta)
{
    static_assert(S::B == 8 && S::K <= 2, "tables for one or two 8-bit codebooks");
    constexpr int K = S::K;
    constexpr int NG = kLutGroups<K>;  // groups of the CTA
    constexpr int NSLOT = NG / 32;     // group slots per lane: 2 (2x8) or 4 (1x8)
    static_assert(NG * S::kChunkBytes == kLutTileBytes, "one kilobyte of codes per row tile");
    extern __shared__ __align__(16) uint8_t lut_smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(lut_smem);  // [256][64] words, see above
    __shared__ uint4 scb[K * 256];     // the codebooks, row k*256 + c
    __shared__ uint4 xs[NG];           // activations of the CTA's groups
    __shared__ uint32_t s_max[2];      // largest |C|, |x| (binary16 bits)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G0 = blockIdx.y * NG;
    const int rt0 = blockIdx.x * rt_per_cta;
    const int rt1 = min(L.rtiles, rt0 + rt_per_cta);
    const int ntw = (rt1 - rt0 - warp + kLutWarps - 1) / kLutWarps;  // this warp's tiles warp + 16 i
    uint8_t *ring = lut_smem + kLutBytes + warp * (kLutRing * kLutTileBytes);

    // codes of this warp's tile i into ring slot i % kLutRing: the tile's
    // kilobyte for the CTA's groups, zero past the padded groups or rows
    auto copy_tile = [&](int i) {
        const int rt = rt0 + warp + kLutWarps * i;
        const bool tile_live = i < ntw && rt < rt1;
        const uint8_t *src = packed + ((size_t)rt * L.gp + G0) * S::kChunkBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int off = h * 512 + lane * 16;
            const bool live = tile_live && G0 + off / S::kChunkBytes < L.gp;
            cp_async16(smem_u32(ring + (i % kLutRing) * kLutTileBytes + off), live ? src + off : packed,
                       live ? 16u : 0u);
        }
    };
    // weights before the dependency wait: codebooks, the first tiles' codes,
    // and the rest of the CTA's codes into L2
    uint4 cw = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x < K * 256) cw = ldg_stream_v4(cb + threadIdx.x);
#pragma unroll
    for (int i = 0; i < kLutRing; ++i) {
        copy_tile(i);
        cp_async_commit();
    }
    {
        const int ngl = min(NG, L.gp - G0);  // groups of this split in the padded layout
        for (int rt = rt0 + kLutWarps * kLutRing + (int)threadIdx.x; rt < rt1; rt += kLutThreads)
            prefetch_l2_bulk(packed + ((size_t)rt * L.gp + G0) * S::kChunkBytes, (uint32_t)(ngl * S::kChunkBytes));
    }
    if (threadIdx.x < 2) s_max[threadIdx.x] = 0;
    prefetch_range_scales(L, scales, rt0 * 8, (rt1 - rt0) * 8);
    grid_dependency_wait();  // x, y and the workspace follow the previous launch
    grid_launch_dependents();
    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x < NG) {
        const int g = G0 + threadIdx.x;
        if (g < L.G) xv = ldg_nc_v4(x + (size_t)g * 8);
        xs[threadIdx.x] = xv;
    }
    if (threadIdx.x < K * 256) scb[threadIdx.x] = cw;
    {
        const uint32_t mc = __reduce_max_sync(0xffffffffu, absmax_h8_bits(cw));
        const uint32_t mx = __reduce_max_sync(0xffffffffu, absmax_h8_bits(xv));
        __syncthreads();  // s_max cleared by threads 0, 1 before anyone updates it
        if (lane == 0) {
            atomicMax(&s_max[0], mc);
            atomicMax(&s_max[1], mx);
        }
    }
    __syncthreads();
    // entries are bounded by 8 max|x| max|C|; NaN or infinity fails the test
    const float bound = 8.f * __half2float(__ushort_as_half((unsigned short)s_max[0])) *
                        __half2float(__ushort_as_half((unsigned short)s_max[1]));
    const bool exact = !(bound < 65504.f);
    if (!exact) {
        // warp w fills the codeword octets n = w + 16 i (codeword kc = 8 n +
        // 0..7, kc = k*256 + c) for every group of the CTA
        const int gid = lane >> 2, t4 = lane & 3;
        const uint32_t *xw = reinterpret_cast<const uint32_t *>(xs);
        const uint32_t *cbw = reinterpret_cast<const uint32_t *>(scb);
        constexpr int MT = NG / 16;  // group tiles
        uint32_t a[MT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            a[m][0] = xw[(16 * m + gid) * 4 + t4];
            a[m][1] = xw[(16 * m + gid + 8) * 4 + t4];
        }
        int off[4];  // slot s of a store writes word l = gid + off[s]
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2) off[s2] = 8 * ((t4 + s2) & 3);
        constexpr int NOCT = K * 256 / 8;
        for (int n = warp; n < NOCT; n += kLutWarps) {
            const uint32_t b0 = cbw[(8 * n + gid) * 4 + t4];
#pragma unroll
            for (int qq = 0; qq < MT / 4; ++qq) {
                // tiles 4 qq + {0, 1} hold groups 64 qq + gid + {0, 8, 16, 24};
                // tiles 4 qq + {2, 3} the same groups + 32
                float lo0[4], lo1[4], hi0[4], hi1[4];
                mma_m16n8k8(lo0, a[4 * qq + 0][0], a[4 * qq + 0][1], b0);
                mma_m16n8k8(lo1, a[4 * qq + 1][0], a[4 * qq + 1][1], b0);
                mma_m16n8k8(hi0, a[4 * qq + 2][0], a[4 * qq + 2][1], b0);
                mma_m16n8k8(hi1, a[4 * qq + 3][0], a[4 * qq + 3][1], b0);
                const int kc = 8 * n + 2 * t4;  // this lane's codewords kc, kc + 1
                // word (c, q, l): c = kc & 255, q = the codebook (2x8) or qq (1x8)
                const int q = (K == 2) ? (kc >> 8) : qq;
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    // v[s] is word l = gid + 8 s: groups (gid + 8 s, + 32) of codeword kc + b
                    const uint32_t v[4] = {f2h2(lo0[b], hi0[b]), f2h2(lo0[2 + b], hi0[2 + b]),
                                           f2h2(lo1[b], hi1[b]), f2h2(lo1[2 + b], hi1[2 + b])};
                    uint32_t r[4], w[4];
#pragma unroll
                    for (int s2 = 0; s2 < 4; ++s2) r[s2] = (t4 & 1) ? v[(s2 + 1) & 3] : v[s2];
#pragma unroll
                    for (int s2 = 0; s2 < 4; ++s2) w[s2] = (t4 & 2) ? r[(s2 + 2) & 3] : r[s2];
                    // w[s2] = v[(t4 + s2) & 3], the word of l = gid + off[s2]
                    uint32_t *dst = lut + ((kc + b) & 255) * 64 + q * 32 + gid;
#pragma unroll
                    for (int s2 = 0; s2 < 4; ++s2) dst[off[s2]] = w[s2];
                }
            }
        }
    }
    __syncthreads();
    const char *lutb = reinterpret_cast<const char *>(lut);
    const uint32_t lane4 = lane * 4;
    float *part = sk.partials + (size_t)blockIdx.y * L.rows8;

    // the tile loop, with the rows' sums from the tables or, when they were
    // skipped, from the exact decode (two copies of the loop, one per case)
    auto tiles = [&](auto exact_tag) {
        constexpr bool kExact = decltype(exact_tag)::value;
        for (int i = 0; i < ntw; ++i) {
            cp_async_wait<kLutRing - 1>();  // tile i has landed (this lane's copies, then every lane's)
            __syncwarp();
            Chunk<S> ch[NSLOT];
            const uint8_t *slot = ring + (i % kLutRing) * kLutTileBytes;
#pragma unroll
            for (int j = 0; j < NSLOT; ++j) {
                const uint8_t *cp = slot + (32 * j + lane) * S::kChunkBytes;
                if constexpr (S::kChunkBytes == 16) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(cp);
                    ch[j].w[0] = v.x, ch[j].w[1] = v.y, ch[j].w[2] = v.z, ch[j].w[3] = v.w;
                } else {
                    const uint2 v = *reinterpret_cast<const uint2 *>(cp);
                    ch[j].w[0] = v.x, ch[j].w[1] = v.y;
                }
            }
            __syncwarp();  // every lane has read the slot
            copy_tile(i + kLutRing);
            cp_async_commit();
            float acc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                if constexpr (!kExact) {
                    __half h[4];
#pragma unroll
                    for (int j = 0; j < NSLOT; ++j)
#pragma unroll
                        for (int k = 0; k < K; ++k) {
                            const int q = (K == 2) ? k : (j >> 1), half = (K == 2) ? j : (j & 1);
                            h[j * K + k] = *reinterpret_cast<const __half *>(
                                lutb + lut_offset<S>(ch[j], r, k, lane4) + q * 128 + half * 2);
                        }
                    acc[r] = __half2float(__hadd(__hadd(h[0], h[1]), __hadd(h[2], h[3])));
                } else {
                    float a = 0.f;
#pragma unroll
                    for (int j = 0; j < NSLOT; ++j) {
                        if (G0 + 32 * j + lane >= L.G) continue;  // a padding group weighs nothing
                        uint4 tm[K];
#pragma unroll
                        for (int k = 0; k < K; ++k) tm[k] = scb[k * 256 + ch[j].code(r, k)];
                        a = dot8(sum_round_fast_h8<K>(tm), xs[32 * j + lane], a);
                    }
                    acc[r] = a;
                }
            }
            const float v = warp_reduce8(acc, lane);
            const int row = (rt0 + warp + kLutWarps * i) * 8 + reduced_row_of_lane(lane);
            if ((lane & 3) == 0) {
                if (gridDim.y == 1) {
                    if (row < L.out) {
                        const float sc = scales ? __half2float(__ushort_as_half(scales[row])) : 1.f;
                        y[row] = __half_as_ushort(__float2half_rn(sc * v));
                    }
                } else {
                    part[row] = v;
                }
            }
        }
    };
    if (exact)
        tiles(std::true_type{});
    else
        tiles(std::false_type{});
    cp_async_wait<0>();
    if (gridDim.y == 1) return;
    // kStaged: the slots are staged in the free tables and code ring (bulk
    // copies); else summed straight from L2, four in flight per float4
    splitk_finish<4>(L, sk, blockIdx.x, gridDim.y, rt0 * 8, (rt1 - rt0) * 8, 1, scales, y,
                     kStaged ? reinterpret_cast<float4 *>(lut_smem) : nullptr, kStaged ? kLutSmem : 0);
}

// ---------------------------------------------------------------------------
// 1x16, batch 1 and 2: codewords into registers, products on the CUDA cores.
//
// At batch 1 or 2 the tensor cores have almost nothing to do and the bound is the
// rate of random 16-byte codeword reads from the 1 MiB codebook.  This kernel
// reads them straight into registers (through L1, which keeps a share of the
// codebook) and multiplies them with x in fp32 (each product of two binary16
// values is exact); it keeps no tile in shared memory, so six CTAs of 128
// threads fit per SM at batch 1 (85 registers; four at batch 2), about 6000
// reads in flight, and L1 keeps most of its capacity for the codebook.
// CTA = 16 row tiles (128 rows) x one split of the groups (128 rows rather
// than 256: half the splits per row range, a shorter split-K finish).  Thread (row tile
// t/8, lane t%8) owns the chunks (its row tile, group G0 + t%8 + 8 j): a
// chunk's 8 codes give the 8 rows' weights of its group.  The first chunk's
// codewords are requested before the CTA waits for the previous launch
// (weights only); then x of the split goes to shared memory as fp32
// ([group][element][batch]), and each row's codeword is replaced by the next
// chunk's as soon as it is used.
// The 8 lanes of a row tile add their row sums with a 3-level
// reduce-scatter; split-K partial sums are finished as for the tables.
// ---------------------------------------------------------------------------
constexpr int kCcThreads = 128;
constexpr int kCcRowTiles = kCcThreads / 8;  // 128 rows per CTA
constexpr int kCcMaxSplits = 32;             // more splits per row range: the tensor-core path
constexpr int kCcMaxBatch = 2;  // measured: faster than the tensor cores at batch 1 and 2, slower from 3
constexpr int kCcStage = 16 * 1024;          // split-K staging (more would take L1 from the codebook)

__device__ __forceinline__ uint32_t cc_code(const uint4 &c, int r)
{
    const uint32_t u = (r < 2) ? c.x : (r < 4) ? c.y : (r < 6) ? c.z : c.w;
    return (u >> (16 * (r & 1))) & 0xffffu;
}

// <w, x> for 8 binary16 weights and 8 fp32 activations (fp32 FMAs)
__device__ __forceinline__ float cc_dot8(float acc, uint4 w, float4 x0, float4 x1)
{
    float2 a = h2f2(w.x);
    acc = fmaf(a.x, x0.x, acc);
    acc = fmaf(a.y, x0.y, acc);
    a = h2f2(w.y);
    acc = fmaf(a.x, x0.z, acc);
    acc = fmaf(a.y, x0.w, acc);
    a = h2f2(w.z);
    acc = fmaf(a.x, x1.x, acc);
    acc = fmaf(a.y, x1.y, acc);
    a = h2f2(w.w);
    acc = fmaf(a.x, x1.z, acc);
    acc = fmaf(a.y, x1.w, acc);
    return acc;
}

// CTAs of the CUDA-core kernel resident per SM, by batch (registers)
template <int NB>
constexpr int kCcPerSMOf = NB == 1 ? 6 : 4;

template <int NB>
__global__ void __launch_bounds__(kCcThreads, kCcPerSMOf<NB>)
gemv_1x16_cc_kernel(Geom L, const uint8_t *__restrict__ packed, const uint4 *__restrict__ cb,
                    const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x,
                    uint16_t *__restrict__ y, SplitK sk, int groups_per_split, int stage_bytes)
{
    // x of the split as fp32, [group][element][batch]; later the finish's staging
    extern __shared__ float4 ccs[];
    float *xs = reinterpret_cast<float *>(ccs);
    const int tid = threadIdx.x, rtl = tid >> 3, gl = tid & 7, lane = tid & 31;
    const int rt = blockIdx.x * kCcRowTiles + rtl;
    const bool rows_live = rt < L.rtiles;
    const int G0 = blockIdx.y * groups_per_split;
    const int ng = min(L.G, G0 + groups_per_split) - G0;
    const int nown = rows_live ? max(0, (ng - gl + 7) / 8) : 0;  // this thread's chunks
    const uint8_t *chunk0 = packed + ((size_t)rt * L.gp + G0 + gl) * 16;  // chunk j at + 128 j
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    // weights only before the dependency wait: the first chunk's codewords
    uint4 code = nown > 0 ? ldg_stream_v4(chunk0) : zero;
    uint4 w[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) w[r] = ldg_nc_v4(cb + cc_code(code, r));
    uint4 next = nown > 1 ? ldg_stream_v4(chunk0 + 128) : zero;
    prefetch_range_scales(L, scales, blockIdx.x * kCcRowTiles * 8, kCcRowTiles * 8);
    grid_dependency_wait();  // x, y and the workspace follow the previous launch
    grid_launch_dependents();
    for (int i = tid; i < ng * 2 * NB; i += kCcThreads) {  // 4 values at a time ([in][batch] is that order)
        const uint2 h = *reinterpret_cast<const uint2 *>(x + (size_t)G0 * 8 * NB + i * 4);
        const float2 a = h2f2(h.x), b = h2f2(h.y);
        ccs[i] = make_float4(a.x, a.y, b.x, b.y);
    }
    __syncthreads();
    float acc[8][NB];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
    for (int j = 0; j < nown; ++j) {
        const float *xg = xs + (gl + 8 * j) * 8 * NB;  // x of this chunk's group
        const uint4 cn = next;
        if (j + 2 < nown) next = ldg_stream_v4(chunk0 + (size_t)(j + 2) * 128);
        const bool more = j + 1 < nown;
        if constexpr (NB == 1) {
            const float4 x0 = reinterpret_cast<const float4 *>(xg)[0], x1 = reinterpret_cast<const float4 *>(xg)[1];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                acc[r][0] = cc_dot8(acc[r][0], w[r], x0, x1);
                if (more) w[r] = ldg_nc_v4(cb + cc_code(cn, r));  // the next chunk's row r
            }
        } else {
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const uint32_t hw[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 wf = h2f2(hw[e]);
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        acc[r][b] = fmaf(wf.x, xg[(2 * e) * NB + b], acc[r][b]);
                        acc[r][b] = fmaf(wf.y, xg[(2 * e + 1) * NB + b], acc[r][b]);
                    }
                }
                if (more) w[r] = ldg_nc_v4(cb + cc_code(cn, r));  // the next chunk's row r
            }
        }
    }
    // reduce-scatter over the 8 lanes of the row tile: lane gl gets row gl
    const int row = rt * 8 + gl;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        float b4[4], b2[2];
        bool hi = lane & 4;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            b4[i] = (hi ? acc[i + 4][b] : acc[i][b]) + __shfl_xor_sync(0xffffffffu, hi ? acc[i][b] : acc[i + 4][b], 4);
        hi = lane & 2;
#pragma unroll
        for (int i = 0; i < 2; ++i)
            b2[i] = (hi ? b4[i + 2] : b4[i]) + __shfl_xor_sync(0xffffffffu, hi ? b4[i] : b4[i + 2], 2);
        hi = lane & 1;
        const float v = (hi ? b2[1] : b2[0]) + __shfl_xor_sync(0xffffffffu, hi ? b2[0] : b2[1], 1);
        if (rows_live && row < L.out) {
            if (gridDim.y == 1) {
                const float sc = scales ? __half2float(__ushort_as_half(scales[row])) : 1.f;
                y[(size_t)row * NB + b] = __half_as_ushort(__float2half_rn(sc * v));
            } else {
                sk.partials[((size_t)blockIdx.y * L.rows8 + row) * NB + b] = v;
            }
        }
    }
    if (gridDim.y == 1) return;
    const int row0 = blockIdx.x * kCcRowTiles * 8;
    splitk_finish(L, sk, blockIdx.x, gridDim.y, row0, min(kCcRowTiles * 8, L.rows8 - row0), NB, scales, y, ccs,
                  stage_bytes);
}

// ---------------------------------------------------------------------------
// 1x16 and 2x8 at decode batches: weights decoded straight into mma.sync
// register fragments.
//
// At batch 2..16 the tensor work of a decode-time product is tiny; what
// costs is producing the weights.  This kernel never stores a decoded tile:
// each warp decodes its weights in registers, in the layout of the A
// operand of mma.sync m16n8k16 (binary16 in, fp32 accumulators), and
// multiplies them there.  The contraction index is permuted so that the
// four k-slots a lane holds in each half of the A fragment are four
// consecutive weights of one group: lane (gid, t4) holds rows gid and
// gid + 8 (two 8-row tiles), group t4 of a set of four groups, weights
// 4h..4h+3 in half h.  So one 16-byte codeword per row and group feeds both
// halves, and the B fragments (the activations) follow the same
// permutation, prebuilt once per CTA in shared memory.
//  * 1x16: the codeword is read straight into registers through L1
//    (ld.global.nc), kRfAhead sets ahead, as the batch-1 CUDA-core path
//    does; the bound is the rate of these random reads.
//  * 2x8: the two codewords come from 8 replicas of the codebooks in
//    shared memory (lane l reads replica l % 8, so the eight lanes of a
//    16-byte access phase never conflict) and are added with one binary16
//    rounding (the exact decode).
// Codes: each warp copies quads of four sets (2 row tiles x 16 groups, one
// 16-byte chunk per lane) into a ring of its own in shared memory with
// cp.async, kRfRing quads in flight, and reads each lane's code from there.
// CTA = 8 warps x 16 rows = 128 rows x `gc` groups; grid = (row blocks,
// group splits); splits are finished by the last CTA of the row block.
// Codes, codebooks and (1x16) the first codewords are requested before the
// CTA waits for the previous launch; activations, outputs and the workspace
// after it.
// ---------------------------------------------------------------------------
constexpr int kRfRing = 3;              // quads of code chunks per warp ring
constexpr int kRfAhead = 4;             // 1x16: sets whose codewords are requested ahead
constexpr int kRfMaxGroups = 256;       // groups per CTA (activation fragments in shared memory)

// 2x8: one CTA of 16 warps per SM, so that the 64 KiB of codebook
// replicas are built once per SM; 1x16: two CTAs of 8 warps per SM.
template <class S>
struct RfTraits {
    static constexpr bool kReplicas = (S::K == 2 && S::B == 8);  // 8 replicas of both codebooks
    static constexpr int kBookBytes = kReplicas ? 8 * S::K * 256 * 16 : 0;
    static constexpr int kWarps = kReplicas ? 16 : 8;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kRows = 16 * kWarps;  // rows per CTA
    static constexpr int kPerSM = kReplicas ? 1 : 2;
};

// bytes of dynamic shared memory: codebook replicas, per-warp code rings,
// activation fragments of the CTA's groups (the kernel works in quads of
// 16 groups, so a split of gc groups has fragments for gc rounded up to 16)
template <class S, int NT>
__host__ __device__ constexpr int rf_smem_bytes(int gc)
{
    return RfTraits<S>::kBookBytes + RfTraits<S>::kWarps * kRfRing * 512 + (gc + 15) / 16 * 16 * 128 * NT;
}

// D += A(16x16, row) * B(16x8, col), binary16 in, fp32 accumulate.
__device__ __forceinline__ void mma_m16n8k16(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint16_t lds_u16(uint32_t addr)
{
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

template <class S, int NT>
__global__ void __launch_bounds__(RfTraits<S>::kThreads, RfTraits<S>::kPerSM)
gemv_rf_kernel(Geom L, const uint8_t *__restrict__ packed, const uint4 *__restrict__ cb,
               const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x, int batch,
               uint16_t *__restrict__ y, SplitK sk, int gc, int smem_bytes)
{
    static_assert(S::kChunkBytes == 16, "16-bit packed words (1x16, 2x8)");
    constexpr bool kRep = RfTraits<S>::kReplicas;
    extern __shared__ __align__(16) uint8_t rf_smem[];
    uint4 *rep = reinterpret_cast<uint4 *>(rf_smem);                        // [K*256][8] replicas
    uint4 *rings = reinterpret_cast<uint4 *>(rf_smem + RfTraits<S>::kBookBytes);  // [warp][kRfRing][32]
    constexpr int kRfThreads = RfTraits<S>::kThreads, kRfRows = RfTraits<S>::kRows;
    uint2 *xfrag = reinterpret_cast<uint2 *>(rf_smem + RfTraits<S>::kBookBytes + RfTraits<S>::kWarps * kRfRing * 512);
    // xfrag: [set][half][NT][32] B fragments

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, t4 = lane & 3;
    const int ta = blockIdx.x * (kRfRows / 8) + 2 * warp;  // this warp's row tiles ta, ta + 1
    const int G0 = blockIdx.y * gc;
    const int ng = min(gc, L.G - G0);   // groups of this split (gc is a multiple of 4)
    const int G1 = G0 + ng;              // groups at or past this one belong to the next split
    const int nquads = (ng + 15) / 16;
    const int nsets = 4 * nquads;

    // code quad q of this warp into ring slot q % kRfRing: lane l copies chunk
    // (row tile ta + l / 16, group G0 + 16 q + l % 16); zeros past the layer
    uint4 *ring = rings + warp * (kRfRing * 32);
    auto copy_quad = [&](int q) {
        const int rt = ta + (lane >> 4), g = G0 + 16 * q + (lane & 15);
        const bool live = q < nquads && rt < L.rtiles && g < G1;
        const uint8_t *src = live ? packed + ((size_t)rt * L.gp + g) * 16 : packed;
        cp_async16(smem_u32(ring + (q % kRfRing) * 32 + lane), src, live ? 16u : 0u);
    };
    // this lane's 16-bit code words of set s (rows gid of tiles ta, ta + 1)
    const uint32_t ring_base = smem_u32(ring);
    auto codes_of = [&](int s, uint32_t &wa, uint32_t &wb) {
        const int q = s >> 2, sl = s & 3;
        const uint32_t a = ring_base + (q % kRfRing) * 512 + (4 * sl + t4) * 16 + gid * 2;
        wa = lds_u16(a);
        wb = lds_u16(a + 16 * 16);
    };

#pragma unroll
    for (int q = 0; q < kRfRing; ++q) {
        copy_quad(q);
        cp_async_commit();
    }
    if constexpr (kRep) {
        // 8 replicas of both codebooks: replica r of codeword kc at slot
        // 8 kc + r; consecutive threads fill consecutive slots, so the stores
        // never conflict (the 8 reads of one codeword hit L1)
        for (int i = threadIdx.x; i < S::K * 256 * 8; i += kRfThreads) rep[i] = ldg_nc_v4(cb + (i >> 3));
    }
    uint4 gw[kRfAhead][2];  // 1x16: codewords of sets s .. s + kRfAhead - 1 (rows gid of ta, ta + 1)
    if constexpr (!kRep) {
        // quads 0 and 1 landed (this lane's copies, then every lane's)
        cp_async_wait<kRfRing - 2>();
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kRfAhead; ++i) {
            uint32_t wa, wb;
            codes_of(i, wa, wb);
            gw[i][0] = ldg_nc_v4(cb + wa);
            gw[i][1] = ldg_nc_v4(cb + wb);
        }
    }
    prefetch_range_scales(L, scales, blockIdx.x * kRfRows, kRfRows);
    grid_dependency_wait();  // x, y and the workspace follow the previous launch
    grid_launch_dependents();
    {
        // B fragments straight from x: entry (s, h, nt, lane (gid, t4)) holds
        // x rows 8 (G0 + 4 s + t4) + 4 h + {0, 1} and {2, 3} of column
        // nt * 8 + gid (zero past the batch or the layer), every load of a
        // thread in flight at once
        if (batch % 8 == 0) {
            // the four x rows of an entry's column block are 16-byte loads:
            // item (s, h, nt, t4) reads rows 8 g + 4 h + j, j < 4, columns
            // nt * 8 .. + 7, and writes the entries of its eight lanes gid
            const int nitem = nsets * 2 * NT * 4;
            for (int it = threadIdx.x; it < nitem; it += kRfThreads) {
                const int t4i = it & 3, nt = (it >> 2) % NT, h = (it >> 2) / NT % 2, st = (it >> 2) / NT / 2;
                const int g = G0 + 4 * st + t4i;
                uint4 r[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    r[j] = g < G1 ? ldg_nc_v4(x + ((size_t)8 * g + 4 * h + j) * batch + nt * 8)
                                   : make_uint4(0u, 0u, 0u, 0u);
                uint2 *dst = xfrag + ((st * 2 + h) * NT + nt) * 32 + t4i;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t v[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[j] = (u4_at(r[j], c >> 1) >> (16 * (c & 1))) & 0xffffu;
                    dst[4 * c] = make_uint2(v[0] | (v[1] << 16), v[2] | (v[3] << 16));
                }
            }
        } else {
            const int nent = nsets * 2 * NT * 32;
            for (int e = threadIdx.x; e < nent; e += kRfThreads) {
                const int ln = e & 31, nt = (e >> 5) % NT, h = (e >> 5) / NT % 2, st = (e >> 5) / NT / 2;
                const int n = nt * 8 + (ln >> 2), g = G0 + 4 * st + (ln & 3);
                const bool live = n < batch && g < G1;
                const uint16_t *xp = x + ((size_t)8 * g + 4 * h) * batch + n;
                uint32_t v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) v[j] = live ? (uint32_t)__ldg(xp + j * batch) : 0u;
                xfrag[e] = make_uint2(v[0] | (v[1] << 16), v[2] | (v[3] << 16));
            }
        }
        __syncthreads();  // also publishes the codebook replicas
    }

    float d[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) d[nt][j] = 0.f;
    const uint32_t xfrag_base = smem_u32(xfrag);
    for (int q = 0; q < nquads; ++q) {
        // quads q and q + 1 of this warp have landed
        cp_async_wait<kRfRing - 2>();
        __syncwarp();
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) {
            const int s = 4 * q + sl;
            uint4 wrow[2];  // decoded weights of rows gid (tile ta) and gid (tile ta + 1), group t4 of set s
            const bool glive = G0 + 4 * s + t4 < G1;  // groups past the split weigh nothing here
            if constexpr (kRep) {
                uint32_t wa, wb;
                codes_of(s, wa, wb);
                const uint32_t c[2] = {wa, wb};
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const uint4 t0 = rep[8 * (c[t] & 0xffu) + (lane & 7)];
                    const uint4 t1 = rep[8 * (256u + (c[t] >> 8)) + (lane & 7)];
                    wrow[t] = add_round_h8(t0, t1);
                }
            } else {
                wrow[0] = gw[sl % kRfAhead][0];
                wrow[1] = gw[sl % kRfAhead][1];
                const int sn = s + kRfAhead;  // its codewords are requested now (codes are in quads q, q + 1)
                if (sn < nsets) {
                    uint32_t wa, wb;
                    codes_of(sn, wa, wb);
                    gw[sl % kRfAhead][0] = ldg_nc_v4(cb + wa);
                    gw[sl % kRfAhead][1] = ldg_nc_v4(cb + wb);
                }
            }
            if (!glive) wrow[0] = wrow[1] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t a[4] = {u4_at(wrow[0], 2 * h), u4_at(wrow[1], 2 * h), u4_at(wrow[0], 2 * h + 1),
                                       u4_at(wrow[1], 2 * h + 1)};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint32_t b0, b1;
                    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                                 : "=r"(b0), "=r"(b1)
                                 : "r"(xfrag_base + (uint32_t)((((s * 2 + h) * NT + nt) * 32 + lane) * 8)));
                    mma_m16n8k16(d[nt], a, b0, b1);
                }
            }
        }
        __syncwarp();  // every lane is done with slot q % kRfRing
        copy_quad(q + kRfRing);
        cp_async_commit();
    }
    cp_async_wait<0>();

    // rows gid of tiles ta, ta + 1; columns nt * 8 + 2 t4 + {0, 1}
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int rt = ta + t, row = rt * 8 + gid;
        if (rt >= L.rtiles) continue;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int col = nt * 8 + 2 * t4 + j;
                if (col >= batch) continue;
                const float v = d[nt][2 * t + j];
                if (gridDim.y == 1) {
                    if (row < L.out) {
                        const float sc = scales ? __half2float(__ushort_as_half(scales[row])) : 1.f;
                        y[(size_t)row * batch + col] = __half_as_ushort(__float2half_rn(sc * v));
                    }
                } else {
                    sk.partials[((size_t)blockIdx.y * L.rows8 + row) * batch + col] = v;
                }
            }
    }
    if (gridDim.y == 1) return;
    const int row0 = blockIdx.x * kRfRows;
    // everything past the replicas stages the finish (the launch sizes the
    // shared memory so that a row block's partial sums fit in one pass)
    const int stage_bytes = smem_bytes - RfTraits<S>::kBookBytes;
    splitk_finish(L, sk, blockIdx.x, gridDim.y, row0, min(kRfRows, L.rows8 - row0), batch, scales, y,
                  reinterpret_cast<float4 *>(rings), stage_bytes);
}

// ---------------------------------------------------------------------------
// Small-batch product on the tensor cores (any batch for 1x16, batch 2..16
// for 2x8), warp-specialised.
//
// Work split, one of two (a template flag): the units of work are (row
// tile m of 128 rows, stage s of 64 input features).
//  * per row tile (kSK false): CTA (m, q) takes stages [q len, (q + 1) len)
//    of row tile m; grid (row tiles, splits).
//  * stream-K (kSK true): units m-major, CTA c takes the `len` units from
//    c len on, so every CTA does the same number of stages whatever the
//    shape; len <= stages per row tile, so a CTA covers the end of one row
//    tile and at most the start of the next: one fp32 TMEM accumulator of 16
//    columns per row tile (segment).  It balances shapes whose row tiles
//    split badly over the SMs (28672 x 8192: 224 tiles of 128 stages).
// A row tile covered by several CTAs is finished by the last to arrive,
// which adds the partial sums in split (CTA) order.
// 4 decoder warps + 1 MMA warp.
// Per stage of 64 input features (8 groups), decoder thread t owns code chunk
// (row tile t/8, group t%8) of the 128 x 64 A tile (128-byte swizzle,
// K-major):
//  * 1x16: the chunk's 8 codewords are the weights; they go straight from
//    the L2-resident codebook into the A tile with 16-byte cp.async, several
//    stages ahead, without holding registers;
//  * 2x8: the two codewords per weight group are read from the codebooks in
//    shared memory and summed with binary16 adds (one rounding), then stored.
// x rows of the stage go straight into the B tile when a row is 16 or 32
// bytes (MN-major, 32-byte swizzle, 16 columns zero-padded), else as raw rows
// into the stage's x slot.  A decoder never waits for another: once its own
// copies of stage j have landed it fences them to the async proxy and arrives
// on full[j].  The MMA warp waits on full[j], builds the B tile from the x
// slot if needed, and one lane issues four tcgen05.mma (M 128, N 16, K 16)
// into the fp32 TMEM accumulator and commits to empty[j] (the decoders'
// signal that the buffer may be refilled) and, after the last stage, to
// acc_full.  Every wait is bounded.
// ---------------------------------------------------------------------------
constexpr int kTcDecoders = 128;
constexpr int kTcThreads = kTcDecoders + 32;
constexpr int kTcBM = 128;
constexpr int kTcN = 16;
// Ring depth and copy lag: 1x16 codewords arrive by cp.async from L2 (a
// 6-stage ring, copies of four stages in flight, which still fits two CTAs
// per SM beside a 3-slot activation ring: the second CTA is what lets
// consecutive launches overlap on an SM, worth more than a deeper ring in a
// lone CTA); the other schemes decode in registers, so only the x copies
// are asynchronous.
template <class S> struct TcRing {
    static constexpr bool kAsyncWeights = (S::K == 1 && S::B == 16);
    // 8-bit codebooks of one or two books are held as 8 replicas, replica r
    // of codeword c at 16-byte slot 8c + r: decoder lane gi reads replica
    // gi, so the 8 lanes of a 16-byte load phase (gi = 0..7) hit 8 distinct
    // bank quads whatever their codes (random codes would conflict ~2.5x).
    // Their 64 KiB leave room for a 2-stage ring at two CTAs per SM.
    static constexpr int kReplicas = (S::kBooksInSmem && S::K <= 2) ? 8 : 1;
    static constexpr int depth = kAsyncWeights ? 6 : (kReplicas > 1 ? 2 : 3), lag = kAsyncWeights ? 4 : 1;
    // 1x16: the decoders only gather weights and start before the previous
    // launch ends; the MMA warp waits for it and loads the activations (B
    // tiles, raw x slots) into a ring of their own, xpre stages ahead into
    // slots last used xring - xpre stages earlier.  Other schemes: the
    // decoders wait, then load each stage's x into the slot of their A
    // buffer (their stage period is set by decode, and a shallow x ring on
    // the MMA warp would put the x latency on its path).
    static constexpr bool kXByMma = kAsyncWeights;
    static constexpr int xring = kXByMma ? 3 : depth, xpre = 2;
};
constexpr int kTcTileA = kTcBM * 64 * 2;  // 16 KiB
constexpr int kTcTileB = 64 * 32;         // 2 KiB: 64 rows x 16 columns
constexpr int kTcXSlot = 64 * 16 * 2;     // raw x rows of one stage, batch <= 16
constexpr int kTcTmemCols = 32;  // two accumulators of 16 columns (row tiles ma, ma + 1)

// Stream-K bookkeeping shared by the kernel and the host plan: row tile m
// owns units [m nst, (m + 1) nst); CTA c owns [c len, (c + 1) len).
struct TcSplit {
    int nst, len;
    __host__ __device__ int first_cta(int m) const { return (m * nst) / len; }
    __host__ __device__ int segments(int m) const { return ((m + 1) * nst - 1) / len - first_cta(m) + 1; }
};
constexpr int kCodeAhead = 4;             // code chunks requested this many stages ahead

template <class S, bool kSK>
__global__ void __launch_bounds__(kTcThreads)
gemv_tc_kernel(Geom L, const uint8_t *__restrict__ packed, const uint4 *__restrict__ cb,
               const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x, int batch,
               uint16_t *__restrict__ y, SplitK sk, void *ws, int len)
{
    constexpr int R = TcRing<S>::depth, LAG = TcRing<S>::lag;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *tileA = smem;                    // [R][16 KiB]
    constexpr int RX = TcRing<S>::xring, PRE = TcRing<S>::xpre;
    uint8_t *tileB = tileA + R * kTcTileA;    // [RX][2 KiB]
    uint8_t *xring = tileB + RX * kTcTileB;   // [RX][2 KiB] raw x rows
    uint4 *scb = reinterpret_cast<uint4 *>(xring + RX * kTcXSlot);  // B = 8 codebooks
    constexpr int NR = TcRing<S>::kReplicas;
    uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(scb) + S::kSmemBookBytes * NR);
    uint64_t *empty = full + R;
    uint64_t *emptyx = empty + R;          // [RX] activation slot free
    uint64_t *acc_full = emptyx + RX;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    uint32_t *abort_flag = tmem_slot + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nst = (L.G + 7) / 8;  // 64-feature stages per row tile
    const TcSplit split{nst, len};
    const int mtiles = (L.out + kTcBM - 1) / kTcBM;
    int ma, sa, nloc, brk;  // first row tile, its first stage, stages, local stage of row tile ma + 1
    if constexpr (kSK) {
        const int u0 = blockIdx.x * len;
        nloc = min(len, mtiles * nst - u0);  // >= 1: the grid ends at the last unit
        ma = u0 / nst;
        sa = u0 - ma * nst;
        brk = nst - sa;
    } else {
        ma = blockIdx.x;
        sa = blockIdx.y * len;
        nloc = min(len, nst - sa);  // >= 1: the grid ends at the last split
        brk = nloc;
    }
    const int nseg = (kSK && brk < nloc) ? 2 : 1;
    // row tile and stage of local stage i
    auto tile_of = [&](int i) { return (kSK && i >= brk) ? ma + 1 : ma; };
    auto stage_of = [&](int i) { return (kSK && i >= brk) ? i - brk : sa + i; };
    // partial-sum slots of row tile m, and this CTA's slot
    auto segments = [&](int m) { return kSK ? split.segments(m) : (int)gridDim.y; };
    auto slot_of = [&](int m) { return kSK ? (int)blockIdx.x - split.first_cta(m) : (int)blockIdx.y; };
    const bool x_direct = (batch == 16 || batch == 8);

    if (S::B == 16 && tid == 0) prefetch_table_share(cb, (uint32_t)S::K * 65536u * 16u);
    if constexpr (S::kBooksInSmem)
        for (int i = tid; i < S::K * 256 * NR; i += kTcThreads) scb[i] = cb[i / NR];
    if (tid == 0) {
        for (int s = 0; s < R; ++s) {
            mbar_init(&full[s], kTcDecoders);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < RX; ++s) {
            mbar_init(&emptyx[s], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTcTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile uint32_t *abort_v = abort_flag;

    if (warp < kTcDecoders / 32) {
        // ------------------------------ decoders ------------------------------
        const int rt_l = tid >> 3, gi = tid & 7;  // A role: 8-row tile within the 128 rows, group
        // code chunk of local stage q for this thread, zero past the end
        auto fetch = [&](int q) {
            const int rt = tile_of(q) * (kTcBM / 8) + rt_l, g = stage_of(q) * 8 + gi;
            return load_chunk<S>(packed, (size_t)rt * L.gp + g, q < nloc && rt < L.rtiles && g < L.G);
        };
        Chunk<S> code_ring[kCodeAhead];
#pragma unroll
        for (int q = 0; q < kCodeAhead; ++q) code_ring[q] = fetch(q);
        // 1x16 decoders touch weights only (codes, codebook): they do not
        // wait for the previous launch on the stream, so their gathers may
        // overlap its end (the MMA warp waits before it loads x, and every
        // store of partial sums or y follows the MMAs).  Other decoders also
        // load x, so they wait first.
        if constexpr (!TcRing<S>::kXByMma) grid_dependency_wait();
        grid_launch_dependents();
        const int kr = tid >> 1, hb = tid & 1;  // x role (other schemes): feature row, 8-column half
        bool ok = true;
        int published = 0;  // this thread has arrived on full[] for stages below this
        // stage loop unrolled by the code-ring depth so every ring index is static
        for (int i0 = 0; ok && i0 < nloc + LAG; i0 += kCodeAhead) {
#pragma unroll
            for (int u = 0; u < kCodeAhead; ++u) {
                const int i = i0 + u;
                if (i >= nloc + LAG) break;
                if (i < nloc) {
                    const int s = stage_of(i), buf = i % R;
                    // the buffer is free once the MMAs of stage i - R completed.
                    // If they have not, the MMA warp is behind (at the start,
                    // it waits for the previous launch): publish every stage
                    // issued so far before blocking, so that it can run them
                    // back to back once it starts.
                    if (i >= R) {
                        const uint32_t par = ((i / R) - 1) & 1;
                        if (!mbar_test_wait(&empty[buf], par)) {
                            cp_async_wait<0>();
                            fence_proxy_async_smem();
                            for (; published < i; ++published) mbar_arrive(&full[published % R]);
                            if (!mbar_wait_ns(&empty[buf], par, kWaitNs)) *abort_v = 1;
                        }
                    }
                    if (*abort_v) {
                        ok = false;
                        break;
                    }
                    const Chunk<S> code = code_ring[u];
                    code_ring[u] = fetch(i + kCodeAhead);
                    const bool live = tile_of(i) * (kTcBM / 8) + rt_l < L.rtiles && s * 8 + gi < L.G;
                    uint8_t *A = tileA + buf * kTcTileA;
                    if constexpr (TcRing<S>::kAsyncWeights) {
                        const uint32_t a0 = smem_u32(A);
#pragma unroll
                        for (int r = 0; r < 8; ++r)
                            cp_async16(a0 + sw128(rt_l * 8 + r, gi),
                                       live ? (const void *)(cb + code.code(r, 0)) : (const void *)cb, live ? 16u : 0u);
                    } else if constexpr (S::K <= 2) {
                        // every codeword read is issued before the first tile
                        // store: the codebooks and the tile share one shared
                        // array, so a store would otherwise hold back the
                        // next row's reads and serialise the eight rows
                        uint4 t[8][S::K];
#pragma unroll
                        for (int r = 0; r < 8; ++r) {
                            if constexpr (NR > 1) {
#pragma unroll
                                for (int k = 0; k < S::K; ++k) t[r][k] = scb[(k * 256 + code.code(r, k)) * NR + gi];
                            } else {
                                gather_terms<S>(code, r, scb, cb, t[r]);
                            }
                        }
#pragma unroll
                        for (int r = 0; r < 8; ++r)
                            *reinterpret_cast<uint4 *>(A + sw128(rt_l * 8 + r, gi)) =
                                live ? sum_round_fast_h8<S::K>(t[r]) : make_uint4(0, 0, 0, 0);
                    } else {
#pragma unroll
                        for (int r = 0; r < 8; ++r) {
                            uint4 t[S::K];
                            gather_terms<S>(code, r, scb, cb, t);
                            *reinterpret_cast<uint4 *>(A + sw128(rt_l * 8 + r, gi)) =
                                live ? sum_round_fast_h8<S::K>(t) : make_uint4(0, 0, 0, 0);
                        }
                    }
                    if constexpr (!TcRing<S>::kXByMma) {
                        // x rows of this stage into the slot of this A buffer:
                        // straight into the B tile when a row is 16 or 32
                        // bytes, else the raw rows into the x slot
                        if (x_direct) {
                            const int k = s * 64 + kr, n0 = hb * 8;
                            const bool in = k < L.in && n0 < batch;
                            cp_async16(smem_u32(tileB + buf * kTcTileB) + sw32(kr, hb),
                                       in ? (const void *)(x + (size_t)k * batch + n0) : (const void *)x, in ? 16u : 0u);
                        } else if (tid < 8 * batch) {
                            const int valid = max(0, min(64, L.in - s * 64)) * batch * 2;
                            const int nb = max(0, min(16, valid - tid * 16));
                            const uint8_t *src = reinterpret_cast<const uint8_t *>(x + (size_t)s * 64 * batch) + tid * 16;
                            cp_async16(smem_u32(xring + buf * kTcXSlot) + tid * 16,
                                       nb > 0 ? (const void *)src : (const void *)x, (uint32_t)nb);
                        }
                    }
                }
                cp_async_commit();  // one group per iteration (empty in the drain)
                const int j = i - LAG;
                if (j >= published) {
                    // this thread's copies of stage j have landed: publish them
                    cp_async_wait<LAG>();
                    fence_proxy_async_smem();
                    mbar_arrive(&full[j % R]);
                    published = j + 1;
                }
            }
        }
        cp_async_wait<0>();
        // ------------------------------ epilogue ------------------------------
        const bool got = (*abort_v == 0) && mbar_wait_ns(acc_full, 0, kWaitNs);
        if (!got) *abort_v = 1;
        tc_fence_after();
        if (__all_sync(0xffffffffu, got)) {
            for (int e = 0; e < nseg; ++e) {
                const int m = ma + e;
                const int row = m * kTcBM + warp * 32 + lane;  // TMEM lane quarter = warp
                float v[16];
                tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + 16u * e, v);
                if (row < L.out) {
                    if (segments(m) == 1) {
                        const float sc = scales ? __half2float(__ushort_as_half(scales[row])) : 1.f;
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            if (n < batch)
                                y[(size_t)row * batch + n] = __half_as_ushort(__float2half_rn(sc * v[n]));
                    } else {
                        float *p = sk.partials + ((size_t)slot_of(m) * L.rows8 + row) * batch;
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            if (n < batch) p[n] = v[n];
                    }
                }
            }
        }
    } else {
        // ------------------------------ MMA warp ------------------------------
        // x, y and the workspace follow the previous launch on the stream:
        // this warp waits for it, then loads x PRE stages ahead (x rows go
        // straight into the B tile when a row is 16 or 32 bytes, else as raw
        // rows into the slot's x buffer)
        constexpr bool kX = TcRing<S>::kXByMma;
        if constexpr (kX) grid_dependency_wait();
        const uint32_t idesc = make_idesc(kTcBM, kTcN, true);
        auto load_x = [&](int q) {
            const int sx = stage_of(q), xb = q % RX;
            if (x_direct) {
#pragma unroll
                for (int c = lane; c < 128; c += 32) {
                    const int kr = c >> 1, n0 = (c & 1) * 8;
                    const int k = sx * 64 + kr;
                    const bool in = k < L.in && n0 < batch;
                    cp_async16(smem_u32(tileB + xb * kTcTileB) + sw32(kr, c & 1),
                               in ? (const void *)(x + (size_t)k * batch + n0) : (const void *)x, in ? 16u : 0u);
                }
            } else {
                const int valid = max(0, min(64, L.in - sx * 64)) * batch * 2;
                for (int t = lane; t < 8 * batch; t += 32) {
                    const int nb = max(0, min(16, valid - t * 16));
                    const uint8_t *src = reinterpret_cast<const uint8_t *>(x + (size_t)sx * 64 * batch) + t * 16;
                    cp_async16(smem_u32(xring + xb * kTcXSlot) + t * 16, nb > 0 ? (const void *)src : (const void *)x,
                               (uint32_t)nb);
                }
            }
        };
        if constexpr (kX) {
#pragma unroll
            for (int q = 0; q < PRE; ++q) {
                if (q < nloc) load_x(q);
                cp_async_commit();  // one group per stage, empty ones included
            }
        }
        for (int j = 0; j < nloc; ++j) {
            const int buf = j % R, xb = kX ? j % RX : buf;
            if constexpr (kX) {
                // x of stage j + PRE, into a slot whose last MMAs (stage
                // j + PRE - RX) were committed RX - PRE iterations ago
                const int q = j + PRE;
                bool fr = true;
                if (q < nloc && q >= RX) fr = mbar_wait_ns(&emptyx[q % RX], ((q / RX) - 1) & 1, kWaitNs);
                if (!__all_sync(0xffffffffu, fr)) {
                    *abort_v = 1;
                    break;
                }
                if (q < nloc) load_x(q);
                cp_async_commit();
                cp_async_wait<PRE>();  // this lane's copies of stage j have landed
                __syncwarp();           // and every lane's
                fence_proxy_async_smem();
            }
            const bool got = mbar_wait_ns(&full[buf], (j / R) & 1, kWaitNs);
            if (!__all_sync(0xffffffffu, got)) {
                *abort_v = 1;
                break;
            }
            if (__any_sync(0xffffffffu, *abort_v != 0)) break;
            if (!x_direct) {
                // B tile rows from the stage's raw x slot: 64 rows x 2 halves
                const uint16_t *xs = reinterpret_cast<const uint16_t *>(xring + xb * kTcXSlot);
#pragma unroll
                for (int c = lane; c < 128; c += 32) {
                    const int krow = c >> 1, n0 = (c & 1) * 8;
                    uint16_t h[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) h[q] = (n0 + q < batch) ? xs[krow * batch + n0 + q] : (uint16_t)0;
                    *reinterpret_cast<uint4 *>(tileB + xb * kTcTileB + sw32(krow, c & 1)) =
                        make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                tc_fence_after();
                const uint32_t a0 = smem_u32(tileA + buf * kTcTileA);
                const uint32_t b0 = smem_u32(tileB + xb * kTcTileB);
                // the first stage of each row tile starts its accumulator
                const uint32_t acc = tmem + ((kSK && j >= brk) ? 16u : 0u);
                const bool first = (j == 0 || (kSK && j == brk));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = smem_desc_sw128(a0 + ks * 32, 16, 1024);
                    const uint64_t bd = smem_desc(b0 + ks * 512, kTcTileB, 256, kSwizzle32B);
                    mma_f16_ss(acc, ad, bd, idesc, (!first || ks > 0) ? 1u : 0u);
                }
                mma_commit(&empty[buf]);                // A buffer free once these MMAs complete
                if constexpr (kX) mma_commit(&emptyx[xb]);  // and the activation slot
            }
            __syncwarp();
        }
        cp_async_wait<0>();  // no copy of x may still be landing when the CTA ends
        if (lane == 0) mma_commit(acc_full);  // completes when every MMA issued above has
    }
    __syncthreads();
    if (*abort_v) {
        if (tid == 0) {
            record_status(ws, AQ_ERR_TIMEOUT);
            mbar_wait_ns(acc_full, 0, kWaitNs);  // drain the issued MMAs (bounded)
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTcTmemCols);
    // arrive even after a timeout so the counters stay consistent (the
    // status word already tells the caller the output is incomplete)
    for (int e = 0; e < nseg; ++e) {
        const int m = ma + e, ns = segments(m);
        if (ns > 1)
            splitk_finish(L, sk, m, ns, m * kTcBM, min(kTcBM, L.rows8 - m * kTcBM), batch, scales, y,
                          reinterpret_cast<float4 *>(tileA), R * kTcTileA);
    }
}

}  // namespace aqk

namespace aqh {
using namespace aqk;

namespace {

enum Path { kLut = 1, kTensor = 2, kCudaCores = 3, kRegFrag = 4 };

struct GemvPlan {
    Path path;
    int ks;          // splits of the group sum (grid.y; 1 for stream-K)
    int len;         // tensor: stages per CTA
    bool stream_k;   // tensor: stream-K split (else per row tile)
    int rt_per_cta;  // row tiles per CTA (LUT path)
    int cc_smem;     // CUDA-core path: dynamic shared memory (x, then the split-K staging)
    int grid_x;
    int counters;    // arrival counters: LUT row ranges, tensor row tiles
    int slots;       // partial-sum slots per row range (0: no split-K)
    size_t ws_bytes;
};


// Depends on the shape and batch only, so the workspace size can be
// computed on a host without a GPU.
template <class S>
constexpr int tc_smem_bytes();

// CTAs of gemv_tc_kernel that fit on one SM (228 KiB of shared memory, 1 KiB
// reserved per CTA; 160 threads each, far below the thread limit).
int tc_resident_ctas(const Geom &g)
{
    int smem = 0;
    with_scheme(g, [&](auto sch) {
        smem = tc_smem_bytes<decltype(sch)>();
        return cudaSuccess;
    });
    return smem > 0 ? std::max(1, (228 * 1024) / (smem + 1024)) : 1;
}

// Shortest stream-K share: below 4 stages a CTA's fixed costs (prologue,
// pipeline fill and drain, split-K finish) dominate.
constexpr int kTcMinLen = 4;

// Cost of `ctas` CTAs of `len` stages each, `res` of them resident per SM,
// in tenths of the time in which an SM running two CTAs advances both by one
// stage; a model fitted to Llama-2 7B/70B shapes at batch 1..16:
//  * k >= 2 CTAs on an SM share its codeword-read throughput (k len / 2
//    periods); a CTA alone on its SM has half the reads in flight and runs
//    about 1.5x slower per stage;
//  * every wave of CTAs pays about three stages of prologue, pipeline fill
//    and drain and split-K finish;
//  * where the decoders start before the previous launch ends (1x16), fewer
//    than 32 free CTA slots keep the next launch from starting early in
//    them, which exposes the fill and drain (about 1.4 + 0.2 batch stages).
long tc_cost(long ctas, int len, int res, int batch, bool early)
{
    const long per_sm = (ctas + kNumSMs - 1) / kNumSMs;
    const long waves = (per_sm + res - 1) / res;
    const long k_last = per_sm - (waves - 1) * res;
    long cost = (waves - 1) * (5L * res * len + 30) + (k_last == 1 ? 15 : 5 * k_last) * (long)len + 30;
    const long last_wave = ctas - (waves - 1) * res * kNumSMs;
    if (early && (long)res * kNumSMs - last_wave < 32) cost += 14 + 2 * batch;
    return cost;
}

// Group splits of the table path: one per kLutGroups groups.
int lut_splits(const Geom &g)
{
    const int ng = g.K == 1 ? kLutGroups<1> : kLutGroups<2>;
    return (g.G + ng - 1) / ng;
}

// Row tiles per CTA of the table path: as many row ranges as put one CTA
// on each SM in one wave.
int lut_rt_per_cta(const Geom &g)
{
    const int ranges = std::max(1, std::min(g.rtiles, kNumSMs / lut_splits(g)));
    return (g.rtiles + ranges - 1) / ranges;
}

// Workspace of the table path: one partial sum per row and group split.
size_t lut_ws(const Geom &g)
{
    const int ks = lut_splits(g);
    return ks > 1 ? kWsData + (size_t)ks * g.rows8 * sizeof(float) : kWsHeader;
}

// Register-fragment path (1x16 from batch 3, 2x8 from batch 2): groups per
// CTA and group splits.  At most kRfMaxGroups groups per CTA, and few
// enough that two CTAs fit on an SM; about two CTAs per SM in all.
// Returns false when the layer's scheme does not take this path, or when
// the split's partial sums would not fit `cap`.
bool plan_rf(const Geom &g, int batch, size_t cap, GemvPlan &p)
{
    const bool k2 = (g.K == 2 && g.B == 8);
    if (!(k2 || (g.K == 1 && g.B == 16))) return false;
    if (batch < (k2 ? 2 : 3)) return false;
    const int nt = batch <= 8 ? 1 : 2;
    auto smem = [&](int gc) {
        return k2 ? (nt == 1 ? rf_smem_bytes<Scheme<2, 8>, 1>(gc) : rf_smem_bytes<Scheme<2, 8>, 2>(gc))
                  : (nt == 1 ? rf_smem_bytes<Scheme<1, 16>, 1>(gc) : rf_smem_bytes<Scheme<1, 16>, 2>(gc));
    };
    const int rows = k2 ? RfTraits<Scheme<2, 8>>::kRows : RfTraits<Scheme<1, 16>>::kRows;
    const int per_sm_slots = k2 ? RfTraits<Scheme<2, 8>>::kPerSM : RfTraits<Scheme<1, 16>>::kPerSM;
    int gc_max = kRfMaxGroups;  // as many groups as fit the CTAs an SM holds
    while (gc_max > 16 && smem(gc_max) > (per_sm_slots == 1 ? 220 : 113) * 1024) gc_max -= 16;
    const int nrb = (g.rtiles + rows / 8 - 1) / (rows / 8);
    auto ws_of = [&](int gcv) {
        const int ks = (g.G + gcv - 1) / gcv;
        return ks > 1 ? kWsData + (size_t)ks * g.rows8 * batch * sizeof(float) : kWsHeader;
    };
    // the split (groups per CTA, a multiple of 4) whose busiest SM has the
    // least work: CTAs beyond the two slots of every SM form a second wave,
    // and an SM that runs two CTAs takes about twice as long as one with one
    int gc = std::min(gc_max, (g.G + 3) / 4 * 4);
    double best = 0;
    for (int ks = 1; ks <= (g.G + 3) / 4; ++ks) {
        const int gcv = (g.G + ks - 1) / ks;
        const int gc4 = (gcv + 3) / 4 * 4;
        if (gc4 > gc_max || (g.G + gc4 - 1) / gc4 != ks) continue;
        if (gc4 < std::min(32, (g.G + 3) / 4 * 4)) break;  // at least 8 sets per CTA: fixed costs dominate below
        if (ws_of(gc4) > cap || (ks > 1 && nrb > kWsMaxCounters)) continue;
        const long ctas = (long)nrb * ks;
        const long per_sm = (ctas + kNumSMs - 1) / kNumSMs;  // CTAs on the busiest SM
        const double load = (double)per_sm * gc4 + (per_sm > per_sm_slots ? 1e9 : 0);  // groups it works through
        if (best == 0 || load < best) {
            best = load;
            gc = gc4;
        }
        if (ctas > (long)per_sm_slots * kNumSMs) break;
    }
    const int ks = (g.G + gc - 1) / gc;
    if (ws_of(gc) > cap || (ks > 1 && nrb > kWsMaxCounters)) return false;
    p.path = kRegFrag;
    p.len = gc;
    p.ks = ks;
    p.grid_x = nrb;
    p.counters = nrb;
    p.slots = ks > 1 ? ks : 0;
    // shared memory: the kernel's own, or more, so that the last CTA of a
    // row block stages all its splits' partial sums in one pass (one L2
    // round trip), while the CTAs an SM holds still fit
    const size_t stage = (size_t)ks * rows * batch * sizeof(float) + (k2 ? RfTraits<Scheme<2, 8>>::kBookBytes : 0);
    const int cap_smem = (per_sm_slots == 1 ? 220 : 113) * 1024;
    p.cc_smem = std::max(smem(gc), (int)std::min<size_t>(stage, (size_t)cap_smem));
    return true;
}

// `cap`: largest workspace the caller can offer (the no-allocation entry
// point's scratch); the plan lengthens the CTAs' shares until its partial
// sums fit, down to one row tile per CTA (no partials).
GemvPlan plan_gemv(const Geom &g, int batch, size_t cap = ~(size_t)0)
{
    GemvPlan p{};
    const int cc_ranges = (g.rtiles + kCcRowTiles - 1) / kCcRowTiles;
    // 1x16 at batch 1..kCcMaxBatch on the CUDA cores: as many group splits
    // as fill the resident CTA slots in one wave (at most kCcMaxSplits, else
    // too few rows for this path) and at most 1536 / batch groups per split
    // (their x in shared memory)
    const int cc_per_sm = batch == 1 ? kCcPerSMOf<1> : kCcPerSMOf<2>;
    const int cc_ks = std::max(1, std::min((cc_per_sm * kNumSMs) / cc_ranges, (g.G + 7) / 8));
    const size_t cc_ws = cc_ks > 1 ? kWsData + (size_t)cc_ks * g.rows8 * batch * sizeof(float) : kWsHeader;
    if (batch <= kCcMaxBatch && g.K == 1 && g.B == 16 && cc_ks <= kCcMaxSplits &&
        (g.G + cc_ks - 1) / cc_ks * batch <= 1536 && cc_ws <= cap &&
        (cc_ks == 1 || cc_ranges <= kWsMaxCounters)) {
        p.path = kCudaCores;
        p.grid_x = cc_ranges;
        p.len = (g.G + cc_ks - 1) / cc_ks;  // groups per split
        p.ks = (g.G + p.len - 1) / p.len;
        p.counters = p.grid_x;
        p.slots = p.ks > 1 ? p.ks : 0;
        const int nvec = kCcRowTiles * 8 * batch / 4;  // float4 of one row range's partial sums
        p.cc_smem = std::max(p.len * 32 * batch, std::min(kCcStage, p.ks > 1 ? p.ks * nvec * 16 : 0));
    } else if (plan_rf(g, batch, cap, p)) {
        // p is filled in
    } else if (batch == 1 && g.B == 8 && g.K <= 2 && lut_ws(g) <= cap) {
        p.path = kLut;
        p.ks = lut_splits(g);
        // one CTA per SM in one wave: every CTA builds its tables once, and
        // a CTA of the next launch fits beside it, so that it can start early
        p.rt_per_cta = lut_rt_per_cta(g);
        p.grid_x = (g.rtiles + p.rt_per_cta - 1) / p.rt_per_cta;
        p.counters = p.grid_x;
        p.slots = p.ks > 1 ? p.ks : 0;
    } else {
        // the tensor-core path, also for 8-bit codebooks at batch 1 when the
        // table path's partial sums would not fit `cap`
        p.path = kTensor;
        const int mtiles = (g.out + kTcBM - 1) / kTcBM;
        const int nst = (g.G + 7) / 8;
        const long units = (long)mtiles * nst;
        const int res = tc_resident_ctas(g);
        const long slots = (long)res * kNumSMs;
        const bool early = (g.K == 1 && g.B == 16);  // decoders that do not wait for the previous launch
        auto ws_of = [&](int nslots) {
            return nslots > 0 ? kWsData + (size_t)nslots * g.rows8 * batch * sizeof(float) : kWsHeader;
        };
        // a split needs one arrival counter per row tile in the fixed area
        const bool may_split = mtiles <= kWsMaxCounters;
        // per row tile: ks splits of `per` stages (the last may be shorter)
        long best_pt = -1;
        p.stream_k = false;
        p.len = nst;
        p.ks = 1;
        for (int ks = 1; ks <= std::max(1, nst / kTcMinLen); ++ks) {
            const int per = (nst + ks - 1) / ks, kk = (nst + per - 1) / per;
            if (kk < ks) continue;  // same split as a smaller ks
            if (kk > 1 && (!may_split || ws_of(kk) > cap)) break;
            const long c = tc_cost((long)mtiles * kk, per, res, batch, early);
            if (best_pt < 0 || c < best_pt) {
                best_pt = c;
                p.len = per;
                p.ks = kk;
            }
        }
        // stream-K: from the share that fills every resident CTA slot in one
        // wave up to one CTA per SM; a row tile meets at most
        // ceil((nst - 1) / len) + 1 shares
        const int lmin = (int)std::min<long>(nst, std::max<long>(kTcMinLen, (units + slots - 1) / slots));
        const int lmax = (int)std::min<long>(nst, std::max<long>(lmin, (units + kNumSMs - 1) / kNumSMs));
        auto sk_slots = [&](int len) { return len >= nst ? 0 : (nst - 1 + len - 1) / len + 1; };
        long best_sk = -1;
        int sk_len = nst;
        for (int len = lmin; len <= lmax && may_split; ++len) {
            if (ws_of(sk_slots(len)) > cap) continue;
            const long c = tc_cost((units + len - 1) / len, len, res, batch, early);
            if (best_sk < 0 || c < best_sk) {
                best_sk = c;
                sk_len = len;
            }
        }
        // stream-K only on a clear predicted gain (the model favours it by
        // a few percent where the per-tile split measures faster: crossing
        // row tiles costs what the model does not see)
        if (best_sk >= 0 && (best_pt < 0 || best_sk * 100 < best_pt * (early ? 95 : 85))) {
            p.stream_k = true;
            p.len = sk_len;
            p.ks = 1;
            p.slots = sk_slots(sk_len);
            p.grid_x = (int)((units + sk_len - 1) / sk_len);
        } else {
            p.slots = p.ks > 1 ? p.ks : 0;
            p.grid_x = mtiles;
        }
        p.counters = mtiles;
        p.rt_per_cta = kTcBM / 8;
    }
    p.ws_bytes = p.slots > 0 ? kWsData + (size_t)p.slots * g.rows8 * batch * sizeof(float) : kWsHeader;
    return p;
}

// ring of (A tile, B tile, x slot) + codebooks + barriers, TMEM slot, flag
template <class S>
constexpr int tc_smem_bytes()
{
    return 1024 + TcRing<S>::depth * kTcTileA + TcRing<S>::xring * (kTcTileB + kTcXSlot) +
           S::kSmemBookBytes * TcRing<S>::kReplicas + (2 * TcRing<S>::depth + TcRing<S>::xring + 1) * 8 + 16;
}

template <class Kern>
cudaError_t set_smem(Kern k, int bytes)
{
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Launch with programmatic stream serialisation: the kernel's weight-only
// prologue may overlap the tail of the previous kernel on the stream; the
// kernel itself waits (griddepcontrol.wait) before touching x, y or the
// workspace.
// With `pdl` false the launch is an ordinary one: the kernel starts only
// after the previous work on the stream has completed (griddepcontrol.wait
// then returns at once).
template <class... KArgs, class... Args>
cudaError_t launch_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t s,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace

size_t gemv_workspace_bytes(const Geom &g, int batch) { return plan_gemv(g, batch).ws_bytes; }

namespace {

cudaError_t launch_plan(const Geom &g, const GemvPlan &p, const void *packed, const uint16_t *cb,
                        const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y, void *ws,
                        cudaStream_t s, bool pdl)
{
    SplitK sk;
    char *base = reinterpret_cast<char *>(ws);
    sk.counters = reinterpret_cast<unsigned *>(base + kWsHeader);
    sk.partials = reinterpret_cast<float *>(base + kWsData);
    const uint8_t *pk = reinterpret_cast<const uint8_t *>(packed);
    const uint4 *c = reinterpret_cast<const uint4 *>(cb);
    const dim3 grid(p.grid_x, p.ks);
    cudaError_t e = cudaSuccess;
    if (p.path == kCudaCores) {
        auto cc = [&](auto kern) {
            cudaError_t r = set_smem(kern, p.cc_smem);
            if (r != cudaSuccess) return r;
            return launch_pdl(pdl, kern, grid, dim3(kCcThreads), p.cc_smem, s, g, pk, c, scales, x, y, sk, p.len,
                              p.cc_smem);
        };
        static_assert(kCcMaxBatch == 2, "one instantiation per batch on this path");
        e = batch == 1 ? cc(gemv_1x16_cc_kernel<1>) : cc(gemv_1x16_cc_kernel<2>);
    } else if (p.path == kRegFrag) {
        auto rf = [&](auto sch, auto ntc) {
            using S = decltype(sch);
            constexpr int NT = decltype(ntc)::value;
            cudaError_t r = set_smem(gemv_rf_kernel<S, NT>, p.cc_smem);
            if (r != cudaSuccess) return r;
            return launch_pdl(pdl, gemv_rf_kernel<S, NT>, grid, dim3(RfTraits<S>::kThreads), p.cc_smem, s, g, pk, c, scales, x,
                              batch, y, sk, p.len, p.cc_smem);
        };
        using One = std::integral_constant<int, 1>;
        using Two = std::integral_constant<int, 2>;
        if (g.K == 2)
            e = batch <= 8 ? rf(Scheme<2, 8>{}, One{}) : rf(Scheme<2, 8>{}, Two{});
        else
            e = batch <= 8 ? rf(Scheme<1, 16>{}, One{}) : rf(Scheme<1, 16>{}, Two{});
    } else if (p.path == kLut) {
        const int smem = kLutSmem;  // the tables and the code rings
        auto lut = [&](auto sch) {
            using S = decltype(sch);
            if constexpr (S::B == 8 && S::K <= 2) {
                auto go = [&](auto kern) {
                    cudaError_t r = set_smem(kern, smem);
                    if (r != cudaSuccess) return r;
                    return launch_pdl(pdl, kern, grid, dim3(kLutThreads), smem, s, g, pk, c, scales, x, y, sk,
                                      p.rt_per_cta);
                };
                return p.ks > 8 ? go(gemv_lut_kernel<S, true>) : go(gemv_lut_kernel<S, false>);
            } else {
                return cudaErrorInvalidValue;
            }
        };
        e = with_scheme(g, lut);
    } else {
        e = with_scheme(g, [&](auto sch) {
            using S = decltype(sch);
            const int smem = tc_smem_bytes<S>();
            if (p.stream_k) {
                cudaError_t r = set_smem(gemv_tc_kernel<S, true>, smem);
                if (r != cudaSuccess) return r;
                return launch_pdl(pdl, gemv_tc_kernel<S, true>, dim3(p.grid_x), dim3(kTcThreads), smem, s, g, pk, c,
                                  scales, x, batch, y, sk, ws, p.len);
            }
            cudaError_t r = set_smem(gemv_tc_kernel<S, false>, smem);
            if (r != cudaSuccess) return r;
            return launch_pdl(pdl, gemv_tc_kernel<S, false>, dim3(p.grid_x, p.ks), dim3(kTcThreads), smem, s, g, pk, c,
                              scales, x, batch, y, sk, ws, p.len);
        });
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const Geom &g, const void *packed, const uint16_t *cb,
                        const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                        void *ws, cudaStream_t s, bool pdl)
{
    return launch_plan(g, plan_gemv(g, batch), packed, cb, scales, x, batch, y, ws, s, pdl);
}

// ---------------------------------------------------------------------------
// Decode-time product without caller-provided workspace.
//
// The split-K partial sums, arrival counters and status word live in one
// file-scope device array (every GPU that loads this library holds it until
// the process exits).  Host code must not hand the array's name to a kernel:
// on the host it is only a stand-in, so its device address is looked up
// with cudaGetSymbolAddress, the device current, once per device and context.  All
// calls share the array, so calls that overlap on the GPU race; each call
// clears the status word and counters (cudaMemsetAsync on its stream) before
// its kernel starts.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_gemv_scratch[AQ_GEMV_NOALLOC_SCRATCH_BYTES];

namespace {

// The array's device address belongs to one CUDA context.  It is looked up
// once per context (the runtime's primary context of a device, or another
// context the caller made current) and kept with the context's id, which
// the driver never reuses within a process: after cudaDeviceReset, or under
// a different current context, the next call looks the address up again
// instead of using a stale one.  The driver calls are fetched at run time,
// so the library does not link the driver library itself.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Id of the calling thread's current context, or 0 if there is none (or the
// driver lacks the calls).
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
        cudaGetLastError();  // a failed query leaves no sticky error behind
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

constexpr int kMaxDevices = 64;
struct ScratchAddr {
    unsigned long long ctx_id;  // 0: not looked up
    void *ptr;
};
std::mutex g_scratch_mutex;
ScratchAddr g_scratch_addr[kMaxDevices] = {};

cudaError_t scratch_for_current_context(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchAddr &a = g_scratch_addr[dev];
    if (id != 0 && a.ctx_id == id) {
        *out = a.ptr;
        return cudaSuccess;
    }
    // with this device current: the array's address in the current context
    // (this also makes the device's primary context current if none was)
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gemv_scratch);
    if (e != cudaSuccess) return e;
    a.ctx_id = id != 0 ? id : current_context_id();
    a.ptr = p;
    *out = p;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_gemv_noalloc(const Geom &g, const void *packed, const uint16_t *cb,
                                const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                                cudaStream_t s, bool *too_large)
{
    const GemvPlan p = plan_gemv(g, batch, AQ_GEMV_NOALLOC_SCRATCH_BYTES);
    *too_large = p.ws_bytes > AQ_GEMV_NOALLOC_SCRATCH_BYTES;
    if (*too_large) return cudaSuccess;
    void *scratch = nullptr;
    cudaError_t e = scratch_for_current_context(&scratch);
    if (e != cudaSuccess) return e;
    // status word and arrival counters must start at zero; the partials are
    // fully written before they are read
    const size_t clear = p.slots > 0 ? kWsData : kWsHeader;
    e = cudaMemsetAsync(scratch, 0, clear, s);
    if (e != cudaSuccess) return e;
    return launch_plan(g, p, packed, cb, scales, x, batch, y, scratch, s, true);
}

}  // namespace aqh
