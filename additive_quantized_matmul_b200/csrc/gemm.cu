// Prefill product Y = diag(s) W X on the 5th-generation tensor cores (sm_100a).
//
// W is decoded tile by tile from its codes (AQLM wiki entry, "Niveau
// intermédiaire": each group of 8 weights is sum_k C_k[i_k]) straight into
// shared memory in the 128-byte-swizzled K-major layout the tensor core
// reads; X tiles are staged MN-major (128-byte swizzle) next to it; one
// thread issues tcgen05.mma (kind::f16: binary16 operands, fp32 accumulator
// in tensor memory).  Tile: M = 128 rows of W, N = 128 tokens, K = 64 input
// features (8 code groups) per stage, two stages so that decoding stage
// k+1 overlaps the MMAs of stage k.  The epilogue reads the accumulator with
// tcgen05.ld, applies the row scale and rounds to binary16.
//
// Every wait is bounded (wall-clock limit via %globaltimer): on give-up the
// kernel records AQ_ERR_TIMEOUT in the workspace status word, drains what
// it issued (again bounded), frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <type_traits>

#include "scheme.cuh"
#include "tc_common.cuh"

namespace aqk {

constexpr int kBM = 128;           // rows of W per CTA (MMA M)
constexpr int kBN = 128;           // tokens per CTA (MMA N)
constexpr int kBK = 64;            // input features per stage (8 groups)
constexpr int kStages = 2;
constexpr int kGemmThreads = 128;  // 4 warps: decode, stage X, epilogue
constexpr int kTileABytes = kBM * kBK * 2;  // 16 KiB
constexpr int kTileBBytes = kBK * kBN * 2;  // 16 KiB
// ---- kernel -----------------------------------------------------------------

template <class S>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(Geom L, const uint8_t *__restrict__ packed, const uint4 *__restrict__ cb,
               const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x, int T,
               uint16_t *__restrict__ y, void *ws)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
    uint8_t *smem = smem_raw + pad;
    uint8_t *tileA = smem;                                // [2][16 KiB]
    uint8_t *tileB = smem + kStages * kTileABytes;        // [2][16 KiB]
    uint4 *scb = reinterpret_cast<uint4 *>(tileB + kStages * kTileBBytes);  // B = 8 codebooks
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(scb) + S::kSmemBookBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kStages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * kBM;
    const int n0 = blockIdx.y * kBN;

    if constexpr (S::kBooksInSmem)
        for (int i = tid; i < S::K * 256; i += kGemmThreads) scb[i] = cb[i];
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kBN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int nk = (L.in + kBK - 1) / kBK;
    const uint32_t idesc = make_idesc(kBM, kBN);
    const bool vec_x = (T % 8) == 0;
    bool ok = true;

    for (int kt = 0; kt < nk; ++kt) {
        const int st = kt & 1;
        if (kt >= kStages) {
            // the MMAs that read this stage were committed at kt - 2; the
            // outcome is made CTA-uniform before anyone leaves the loop
            const bool got = mbar_wait_ns(&bars[st], ((kt - kStages) / kStages) & 1, kWaitNs);
            if (!__syncthreads_and(got)) { ok = false; break; }
        }
        uint8_t *A = tileA + st * kTileABytes;
        uint8_t *Bt = tileB + st * kTileBBytes;

        // -- decode the W tile: thread -> (row tile rt_l = tid/8, group gi = tid%8)
        {
            const int rt_l = tid >> 3, gi = tid & 7;
            const int rt = (m0 >> 3) + rt_l;
            const int g = kt * 8 + gi;
            const bool live = (rt < L.rtiles) && (g < L.G);
            const Chunk<S> code = load_chunk<S>(packed, (size_t)rt * L.gp + g, live);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (live) {
                    uint4 t[S::K];
                    gather_terms<S>(code, r, scb, cb, t);
                    v = sum_round_fast_h8<S::K>(t);
                }
                const uint32_t row = rt_l * 8 + r;
                *reinterpret_cast<uint4 *>(A + sw128(row, gi)) = v;
            }
        }
        // -- stage the X tile: rows k (input features), 128 tokens as two
        //    64-token MN-major atoms columns of 64 rows x 128 bytes each.
        for (int i = tid; i < kBK * (kBN / 8); i += kGemmThreads) {
            const int k = i / (kBN / 8);
            const int c16 = i % (kBN / 8);      // 16-byte chunk along tokens
            const int nb = c16 >> 3, c = c16 & 7;
            const int gk = kt * kBK + k;
            const int gn = n0 + c16 * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (gk < L.in) {
                const uint16_t *src = x + (size_t)gk * T + gn;
                if (vec_x && gn + 8 <= T) {
                    v = ldg_nc_v4(src);
                } else {
                    uint16_t h[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) h[j] = (gn + j < T) ? src[j] : (uint16_t)0;
                    v = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                                   h[6] | (h[7] << 16));
                }
            }
            *reinterpret_cast<uint4 *>(Bt + nb * (kBK * 128) + sw128(k, c)) = v;
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(A), b0 = smem_u32(Bt);
#pragma unroll
            for (int ks = 0; ks < kBK / 16; ++ks) {
                // A: K-major, +32 bytes per 16-element K step inside the swizzle row
                const uint64_t ad = smem_desc_sw128(a0 + ks * 32, 16, 1024);
                // B: MN-major, 64-token blocks 8 KiB apart (LBO), 8-row K groups
                // 1 KiB apart (SBO), +2 KiB per 16-row K step
                const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, kBK * 128, 1024);
                mma_f16_ss(tmem, ad, bd, idesc, (kt > 0 || ks > 0) ? 1u : 0u);
            }
            mma_commit(&bars[st]);
        }
    }

    // Wait for the last commit (it covers every earlier MMA).
    if (ok && nk > 0) {
        const int last = nk - 1;
        ok = __syncthreads_and(mbar_wait_ns(&bars[last & 1], (last / kStages) & 1, kWaitNs));
    }
    if (!ok) {
        if (tid == 0) record_status(ws, AQ_ERR_TIMEOUT);
        // drain: give the issued MMAs one more bounded chance to finish
        if (nk > 0) mbar_wait_ns(&bars[(nk - 1) & 1], ((nk - 1) / kStages) & 1, kWaitNs);
    }
    tc_fence_after();

    if (ok) {
        // Epilogue: warp w owns TMEM lanes 32w..32w+31 = rows m0 + 32w + lane.
        const int row = m0 + warp * 32 + lane;
        const float sc = (row < L.out && scales) ? __half2float(__ushort_as_half(scales[row])) : 1.f;
        const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < kBN; c0 += 16) {
            float v[16];
            tmem_ld16(tbase + c0, v);
            if (row < L.out) {
                const int gn = n0 + c0;
                uint16_t *dst = y + (size_t)row * T + gn;
                if (vec_x && gn + 16 <= T) {
                    uint4 o0 = make_uint4(f2h2(sc * v[0], sc * v[1]), f2h2(sc * v[2], sc * v[3]),
                                          f2h2(sc * v[4], sc * v[5]), f2h2(sc * v[6], sc * v[7]));
                    uint4 o1 = make_uint4(f2h2(sc * v[8], sc * v[9]), f2h2(sc * v[10], sc * v[11]),
                                          f2h2(sc * v[12], sc * v[13]), f2h2(sc * v[14], sc * v[15]));
                    reinterpret_cast<uint4 *>(dst)[0] = o0;
                    reinterpret_cast<uint4 *>(dst)[1] = o1;
                } else {
                    for (int j = 0; j < 16; ++j)
                        if (gn + j < T) dst[j] = __half_as_ushort(__float2half_rn(sc * v[j]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kBN);
}


// ---- warp-specialised kernel (T a multiple of 8) ---------------------------
//
// Tile M = 128 rows x N = BN tokens (256 or 512), K = 64 per stage; the
// decoded W tile feeds BN tokens, so BN = 512 halves the decode work per
// MMA (the 1x16 decode, ~1024 random L2 gathers per stage, is slower than
// the four N = 256 MMAs of a stage).  Split-K over the input features
// (blockIdx.z) fills the SMs when the tile grid is small.
//   warp 0     X producer: one lane issues BN/64 2-D TMA loads per stage (64
//              tokens x 64 features each, 128-byte swizzle, MN-major) that
//              complete on full_b[stage];
//   warp 1     MMA issuer: one lane waits for full_a/full_b, issues
//              tcgen05.mma (M 128, N 256, K 16; two per K step for BN = 512)
//              into a BN-column fp32 TMEM accumulator and commits to
//              empty[stage] (buffer free) and, after the last stage, to
//              acc_full;
//   warps 2-5  decoders, then epilogue: thread t owns code chunk (row tile
//              t/8, group t%8) of each stage.  1x16: the 8 codewords go from
//              the L2-resident codebook straight into the swizzled A tile by
//              16-byte cp.async, a few stages ahead; 2x8: codewords come from
//              the codebooks in shared memory, summed with binary16 adds.
//              Each thread fences its writes to the async proxy and arrives
//              on full_a[stage] (128 arrivals).  The epilogue reads TMEM lanes
//              32*(warp%4).. with tcgen05.ld, scales, rounds and stores (one
//              split); a split's CTAs finish together (gemm_cluster_finish,
//              gemm_tail_finish).
// Ring depth: 4 stages of (16 KiB A + 32 KiB B) for BN = 256, 3 when the
// 32 KiB of 8x8 codebooks share the shared memory; 2 stages of (16 + 64 KiB)
// for BN = 512.
template <class S, int BN>
constexpr int kWsStagesOf = (BN == 512) ? 2 : (S::kSmemBookBytes > 8192 || (S::K == 1 && S::B == 16)) ? 3 : 4;
// The W (decoded) tiles have a ring of their own, 5 deep (4 with the 32 KiB
// of 8x8 codebooks): with 512-token X tiles taking 64 KiB a stage, a shared
// ring would be 2 deep.  The 1x16 decoders (two groups of 128 threads, two
// of each group's stages in flight: about 4000 codeword reads per CTA) need
// the depth; at 256-token tiles 1x16 trades an X stage for two W stages
// (6 W, 3 X).
template <class S, int BN>
constexpr int kWsAStagesOf = (BN == 512) ? ((S::kSmemBookBytes > 8192) ? 4 : 5)
                                         : ((S::K == 1 && S::B == 16) ? 6 : kWsStagesOf<S, BN>);
// Decoder groups of 4 warps taking alternate stages: one CTA per SM (the X
// tiles fill its shared memory), so the decode rate per SM is that of its
// decoders; with one or two codebooks two groups run (twice the 1x16
// codeword reads in flight; twice the shared-memory decode of 8-bit codes:
// at 512 tokens 20 % faster for both), eight 8-bit codebooks keep one (their
// registers).
template <class S>
constexpr int kWsGroupsOf = (S::K <= 2) ? 2 : 1;
template <class S>
constexpr int kWsThreadsOf = 64 + 128 * kWsGroupsOf<S>;  // X producer, MMA issuer, decoders
constexpr int kWsLag = 2;                     // cp.async stages in flight per decoder (< ring depth)

struct GemmSplit {
    float *partials;  // a split cluster's scratch (gemm_cluster_finish's slices), or null with one split
};

// Split-K finish of a split launched as one thread-block cluster of `ks`
// CTAs along blockIdx.z (ks = 2, 4 or 8; the split index is the CTA's rank).
// The cluster guarantees that the splits of a tile run at the same time, so
// the finish is spread over all of them instead of left to the last one:
// CTA z owns the tile's columns [z BN / ks, (z + 1) BN / ks).  Each CTA
// writes the fp32 sums of the columns it does not own from tensor memory
// to its slice of the split scratch (L2), the cluster barrier publishes
// them, and each CTA adds, for its own columns, every split's sums in split
// order (its own straight from tensor memory), scales, rounds and writes y.
// The scratch holds whole tiles in the order tensor memory hands them out:
// float4 j of column block cb of tile row r at ((cb 4 + j) 128 + r), so a
// warp's 32 rows are 512 contiguous bytes for the writer and the reader
// alike (the owner's thread of a row is the writer's thread of that row).
// `fw` numbers the finishing warps 0 .. NW - 1 (warp & 3 is the TMEM lane
// quarter; NW = 8 splits the columns between two warps per quarter), -1
// for the others.  Every thread of the CTA calls it (the cluster barrier
// needs them all), also after a timeout: then no tensor memory is read and
// the output is incomplete, which the status word reports.
template <int BN, int NW>
__device__ void gemm_cluster_finish(const Geom &L, uint32_t tmem, float *__restrict__ partials, int m0, int n0,
                                    int T, int ks, const uint16_t *__restrict__ scales, uint16_t *__restrict__ y,
                                    int fw, bool ok)
{
    constexpr int kH = NW / 4;  // warps per TMEM lane quarter
    const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
    const int z = (int)blockIdx.z;
    const int cw = BN / ks;  // columns each split owns (a multiple of 16)
    const int r = q * 32 + lane, row = m0 + r;
    // this tile's slices: one per split, kBM x BN floats each
    const size_t tile = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
    float4 *slices = reinterpret_cast<float4 *>(partials) + tile * ks * (kBM * BN / 4);
    constexpr size_t kSlice = kBM * BN / 4;  // float4 per slice
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    tc_fence_after();
    if (fw >= 0 && ok) {
        float4 *mine = slices + (size_t)z * kSlice;
#pragma unroll 1
        for (int c0 = 16 * (fw / 4); c0 < BN; c0 += 16 * kH) {
            if (c0 / cw == z || n0 + c0 >= T) continue;  // warp-uniform
            float v[16];
            tmem_ld16(tq + (uint32_t)c0, v);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                __stcg(mine + ((c0 / 16) * 4 + j) * kBM + r, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        }
        fence_acq_rel_gpu();
    }
    cluster_sync_all();  // every split's sums are in L2
    if (fw < 0 || !ok) return;
    const bool live_row = row < L.out;
    const float sc = (live_row && scales) ? __half2float(__ushort_as_half(scales[row])) : 1.f;
#pragma unroll 1
    for (int c0 = z * cw + 16 * (fw / 4); c0 < (z + 1) * cw; c0 += 16 * kH) {
        const int gn = n0 + c0;
        if (gn >= T) break;  // warp-uniform
        float v[16];
        tmem_ld16(tq + (uint32_t)c0, v);
        const float4 *src = slices + ((c0 / 16) * 4) * kBM + r;
        float acc[16];
        // four splits' loads in flight at a time, added in split order
        for (int z0 = 0; z0 < ks; z0 += 4) {
            float4 t[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (z0 + i < ks && z0 + i != z) t[i][j] = __ldcg(src + (size_t)(z0 + i) * kSlice + j * kBM);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (z0 + i >= ks) break;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 u = (z0 + i == z) ? make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3])
                                                   : t[i][j];
                    if (z0 + i == 0) {
                        acc[4 * j] = u.x, acc[4 * j + 1] = u.y, acc[4 * j + 2] = u.z, acc[4 * j + 3] = u.w;
                    } else {
                        acc[4 * j] += u.x, acc[4 * j + 1] += u.y, acc[4 * j + 2] += u.z, acc[4 * j + 3] += u.w;
                    }
                }
            }
        }
        if (!live_row) continue;
        uint16_t *dst = y + (size_t)row * T + gn;
        const uint4 o0 = make_uint4(f2h2(sc * acc[0], sc * acc[1]), f2h2(sc * acc[2], sc * acc[3]),
                                    f2h2(sc * acc[4], sc * acc[5]), f2h2(sc * acc[6], sc * acc[7]));
        const uint4 o1 = make_uint4(f2h2(sc * acc[8], sc * acc[9]), f2h2(sc * acc[10], sc * acc[11]),
                                    f2h2(sc * acc[12], sc * acc[13]), f2h2(sc * acc[14], sc * acc[15]));
        reinterpret_cast<uint4 *>(dst)[0] = o0;  // T % 8 == 0: gn + 8 <= T
        if (gn + 16 <= T) reinterpret_cast<uint4 *>(dst)[1] = o1;
    }
}

// The tail of a tile grid larger than one wave: when the last wave would
// hold few tiles, their input features are split over `ks` CTAs each (a 1-D
// grid: whole tiles first, then the tail tiles' splits), so the last wave
// fills the SMs.  Such a tile is finished by the last of its splits to
// arrive: each writes its fp32 sums from tensor memory to its slice (the
// order tensor memory hands them out, as gemm_cluster_finish), arrives on
// the tile's counter (acq_rel), and the last adds every split's sums in
// split order (its own from tensor memory; deterministic), scales, rounds,
// writes y and resets the counter.  Every thread of the CTA calls it.
template <int BN, int NW>
__device__ void gemm_tail_finish(const Geom &L, uint32_t tmem, float *__restrict__ slices_base, unsigned *counter,
                                 int m0, int n0, int T, int z, int ks, const uint16_t *__restrict__ scales,
                                 uint16_t *__restrict__ y, int fw, bool ok)
{
    constexpr int kH = NW / 4;
    constexpr size_t kSlice = kBM * BN / 4;  // float4 per slice
    __shared__ unsigned s_last;
    const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
    const int r = q * 32 + lane, row = m0 + r;
    float4 *slices = reinterpret_cast<float4 *>(slices_base);
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    tc_fence_after();
    if (fw >= 0 && ok) {
        float4 *mine = slices + (size_t)z * kSlice;
#pragma unroll 1
        for (int c0 = 16 * (fw / 4); c0 < BN; c0 += 16 * kH) {
            if (n0 + c0 >= T) break;  // warp-uniform
            float v[16];
            tmem_ld16(tq + (uint32_t)c0, v);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                __stcg(mine + ((c0 / 16) * 4 + j) * kBM + r, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // the barrier orders the CTA's slice stores before this increment,
        // whose release publishes them; its acquire orders the last CTA's
        // reads after every split's
        const unsigned prev = atom_add_acq_rel_gpu(counter, 1u);
        s_last = (prev == (unsigned)ks - 1u) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_last) return;
    if (fw >= 0 && ok) {
        const bool live_row = row < L.out;
        const float sc = (live_row && scales) ? __half2float(__ushort_as_half(scales[row])) : 1.f;
#pragma unroll 1
        for (int c0 = 16 * (fw / 4); c0 < BN; c0 += 16 * kH) {
            const int gn = n0 + c0;
            if (gn >= T) break;  // warp-uniform
            float v[16];
            tmem_ld16(tq + (uint32_t)c0, v);
            const float4 *src = slices + ((c0 / 16) * 4) * kBM + r;
            float acc[16];
            for (int z0 = 0; z0 < ks; z0 += 4) {
                float4 t[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (z0 + i < ks && z0 + i != z) t[i][j] = __ldcg(src + (size_t)(z0 + i) * kSlice + j * kBM);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (z0 + i >= ks) break;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float4 u = (z0 + i == z) ? make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3])
                                                       : t[i][j];
                        if (z0 + i == 0) {
                            acc[4 * j] = u.x, acc[4 * j + 1] = u.y, acc[4 * j + 2] = u.z, acc[4 * j + 3] = u.w;
                        } else {
                            acc[4 * j] += u.x, acc[4 * j + 1] += u.y, acc[4 * j + 2] += u.z, acc[4 * j + 3] += u.w;
                        }
                    }
                }
            }
            if (!live_row) continue;
            uint16_t *dst = y + (size_t)row * T + gn;
            const uint4 o0 = make_uint4(f2h2(sc * acc[0], sc * acc[1]), f2h2(sc * acc[2], sc * acc[3]),
                                        f2h2(sc * acc[4], sc * acc[5]), f2h2(sc * acc[6], sc * acc[7]));
            const uint4 o1 = make_uint4(f2h2(sc * acc[8], sc * acc[9]), f2h2(sc * acc[10], sc * acc[11]),
                                        f2h2(sc * acc[12], sc * acc[13]), f2h2(sc * acc[14], sc * acc[15]));
            reinterpret_cast<uint4 *>(dst)[0] = o0;  // T % 8 == 0: gn + 8 <= T
            if (gn + 16 <= T) reinterpret_cast<uint4 *>(dst)[1] = o1;
        }
    }
    if (threadIdx.x == 0) *counter = 0u;
}

// Grid of the tail mode: CTAs [0, full) take whole tiles (tile = index), the
// others split the tiles from `full` on, `ks` CTAs of `per` stages each.
struct TailMap {
    int full;  // CTAs with a whole tile; 0: no tail mode (3-D grid)
    int ks;    // splits per tail tile
    int per;   // 64-feature stages per split
};

template <class S, int BN>
__global__ void __launch_bounds__(kWsThreadsOf<S>, 1)
gemm_ws_kernel(const __grid_constant__ CUtensorMap xmap, Geom L, const uint8_t *__restrict__ packed,
               const uint4 *__restrict__ cb, const uint16_t *__restrict__ scales, int T,
               uint16_t *__restrict__ y, void *ws, GemmSplit sp, int stages_per_split, int cluster_ks, TailMap tm)
{
    constexpr int kWsStages = kWsStagesOf<S, BN>;    // X ring
    constexpr int kWsAStages = kWsAStagesOf<S, BN>;  // W ring
    constexpr int kWsTileB = kBK * BN * 2;   // 32 or 64 KiB
    constexpr int kN = BN < 256 ? BN : 256;  // N of one MMA instruction
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *tileA = smem;                                   // [stages][16 KiB]
    uint8_t *tileB = smem + kWsAStages * kTileABytes;        // [X stages][32 or 64 KiB]
    uint4 *scb = reinterpret_cast<uint4 *>(tileB + kWsStages * kWsTileB);
    uint64_t *full_a = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(scb) + S::kSmemBookBytes);
    uint64_t *full_b = full_a + kWsAStages;
    uint64_t *empty = full_b + kWsStages;       // X buffers free
    uint64_t *empty_a = empty + kWsStages;      // W buffers free
    uint64_t *acc_full = empty_a + kWsAStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    uint32_t *abort_flag = tmem_slot + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the CTA's tile and split: a 3-D grid (row tile, token tile, split), or
    // the tail mode's 1-D grid
    int mt = blockIdx.x, nt = blockIdx.y, z = blockIdx.z, per = stages_per_split, tail_idx = -1;
    if (tm.ks > 0) {
        const int mtiles = (L.out + kBM - 1) / kBM;
        int tile = blockIdx.x;
        z = 0;
        per = (L.in + kBK - 1) / kBK;
        if (tile >= tm.full) {
            const int rr = tile - tm.full;
            tail_idx = rr / tm.ks;
            z = rr % tm.ks;
            tile = tm.full + tail_idx;
            per = tm.per;
        }
        mt = tile % mtiles;
        nt = tile / mtiles;
    }
    const int m0 = mt * kBM;
    const int n0 = nt * BN;
    // this split's stages: global stages s0 .. s0 + nk - 1 (64 features each)
    const int s0 = z * per;
    const int nk = max(0, min((L.in + kBK - 1) / kBK, s0 + per) - s0);
    const int g0 = s0 * 8;  // first code group of the split

    // 1x16: codewords go from L2 into the tile by cp.async, copies of kWsLag
    // stages in flight; other schemes decode in registers
    constexpr bool kAsyncWeights = (S::K == 1 && S::B == 16);
    if (S::B == 16 && tid == 0) prefetch_table_share(cb, (uint32_t)S::K * 65536u * 16u);
    if constexpr (S::kBooksInSmem)
        for (int i = tid; i < S::K * 256; i += kWsThreadsOf<S>) scb[i] = cb[i];
    if (tid == 0) {
        for (int s = 0; s < kWsAStages; ++s) {
            mbar_init(&full_a[s], 128);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < kWsStages; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile uint32_t *abort_v = abort_flag;
    // programmatic dependent launch: before the wait a thread reads weights
    // only (codes, codebooks); X, y, the scales and the workspace follow it
    grid_launch_dependents();

    if (warp == 0) {
        // ---------------- X producer ----------------
        if (lane == 0) {
            grid_dependency_wait();
            for (int s = 0; s < nk; ++s) {
                const int buf = s % kWsStages;
                if (s >= kWsStages && !mbar_wait_ns(&empty[buf], ((s / kWsStages) - 1) & 1, kWaitNs)) {
                    *abort_v = 1;
                    break;
                }
                if (*abort_v) break;
                mbar_arrive_expect_tx(&full_b[buf], kWsTileB);
                const uint32_t dst = smem_u32(tileB + buf * kWsTileB);
#pragma unroll
                for (int q = 0; q < BN / 64; ++q)
                    tma_load_2d(dst + q * (kBK * 128), &xmap, n0 + 64 * q, (s0 + s) * kBK, &full_b[buf]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = make_idesc(kBM, kN, true);
            int s = 0;
            for (; s < nk; ++s) {
                const int buf = s % kWsStages, abuf = s % kWsAStages;
                if (!mbar_wait_ns(&full_a[abuf], (s / kWsAStages) & 1, kWaitNs) ||
                    !mbar_wait_ns(&full_b[buf], (s / kWsStages) & 1, kWaitNs)) {
                    *abort_v = 1;
                    break;
                }
                if (*abort_v) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(tileA + abuf * kTileABytes);
                const uint32_t b0 = smem_u32(tileB + buf * kWsTileB);
#pragma unroll
                for (int ks = 0; ks < kBK / 16; ++ks) {
                    const uint64_t ad = smem_desc_sw128(a0 + ks * 32, 16, 1024);
#pragma unroll
                    for (int h = 0; h < BN / kN; ++h) {
                        // tokens 256 h .. : four 64-token boxes further on
                        const uint64_t bd = smem_desc_sw128(b0 + h * (kN / 64) * (kBK * 128) + ks * 2048, kBK * 128, 1024);
                        mma_f16_ss(tmem + h * kN, ad, bd, idesc, (s > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                mma_commit(&empty[buf]);     // X buffer free once these MMAs complete
                mma_commit(&empty_a[abuf]);  // and the W buffer
            }
            mma_commit(acc_full);  // completes when every MMA issued above has
        }
    } else {
        // ---------------- decoders ----------------
        // group dg takes stages dg, dg + NG, dg + 2 NG, ... (its own stage k
        // is stage dg + NG k); group 0 also runs the epilogue
        constexpr int NG = kWsGroupsOf<S>;
        const int dg = (tid - 64) / 128;
        const int t = (tid - 64) % 128;
        const int nown = (nk - dg + NG - 1) / NG;
        const int rt_l = t >> 3, gi = t & 7;
        const int rt = (m0 >> 3) + rt_l;
        const bool rows_live = rt < L.rtiles;
        // code chunks kCodeAhead stages ahead (register ring): a stage's
        // gathers never wait on an HBM round trip
        constexpr int kCodeAhead = 4;
        Chunk<S> code_ring[kCodeAhead];
#pragma unroll
        for (int q = 0; q < kCodeAhead; ++q) {
            const int sq = dg + NG * q;
            code_ring[q] = load_chunk<S>(packed, (size_t)rt * L.gp + g0 + sq * 8 + gi,
                                         sq < nk && rows_live && g0 + sq * 8 + gi < L.G);
        }
        // copies of kLag stages stay in flight; a stage is published kLag
        // iterations after it is issued, so kLag must stay below the ring
        // depth (the decoder waits for the MMAs of stage s - depth first)
        // (with NG groups a lag of kLag own stages spans NG kLag stages of the ring)
        constexpr int kLag = !kAsyncWeights ? 0 : kWsLag;
        static_assert(NG * kLag < kWsAStages || !kAsyncWeights, "copy lag must leave the MMAs a stage of slack");
        bool ok = true;
        int published = 0;  // own stages below this have been arrived on full_a[]
        // unrolled by the ring depth so every ring index is static
        for (int k0 = 0; ok && k0 < nown + kLag; k0 += kCodeAhead) {
#pragma unroll
            for (int u = 0; u < kCodeAhead; ++u) {
                const int k = k0 + u, s = dg + NG * k;  // own stage, stage
                if (k >= nown + kLag) break;
                if (k < nown) {
                    const int buf = s % kWsAStages;
                    // the buffer is free once the MMAs of stage s - depth
                    // completed; before blocking on it, publish every stage
                    // this thread has issued (the MMAs may need them first)
                    if (s >= kWsAStages) {
                        const uint32_t par = ((s / kWsAStages) - 1) & 1;
                        if (!mbar_test_wait(&empty_a[buf], par)) {
                            if constexpr (kAsyncWeights) {
                                cp_async_wait<0>();
                                fence_proxy_async_smem();
                                for (; published < k; ++published)
                                    mbar_arrive(&full_a[(dg + NG * published) % kWsAStages]);
                            }
                            if (!mbar_wait_ns(&empty_a[buf], par, kWaitNs)) *abort_v = 1;
                        }
                    }
                    if (*abort_v) {
                        ok = false;
                        break;
                    }
                    const Chunk<S> code = code_ring[u];
                    const bool live = rows_live && g0 + s * 8 + gi < L.G;
                    {
                        const int sn = s + NG * kCodeAhead;
                        const int g = g0 + sn * 8 + gi;
                        code_ring[u] = load_chunk<S>(packed, (size_t)rt * L.gp + g, sn < nk && rows_live && g < L.G);
                    }
                    uint8_t *A = tileA + buf * kTileABytes;
                    if constexpr (kAsyncWeights) {
                        const uint32_t a0 = smem_u32(A);
#pragma unroll
                        for (int r = 0; r < 8; ++r)
                            cp_async16(a0 + sw128(rt_l * 8 + r, gi),
                                       live ? (const void *)(cb + code.code(r, 0)) : (const void *)cb, live ? 16u : 0u);
                    } else if constexpr (S::K <= 2) {
                        // all codeword reads before the first tile store (the
                        // books and the tile share one shared array)
                        uint4 t[8][S::K];
#pragma unroll
                        for (int r = 0; r < 8; ++r) gather_terms<S>(code, r, scb, cb, t[r]);
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
                }
                if constexpr (kAsyncWeights) {
                    cp_async_commit();
                    const int j = k - kLag;  // own stage whose copies have landed
                    if (j >= published) {
                        cp_async_wait<kLag>();
                        fence_proxy_async_smem();
                        mbar_arrive(&full_a[(dg + NG * j) % kWsAStages]);
                        published = j + 1;
                    }
                } else {
                    fence_proxy_async_smem();
                    mbar_arrive(&full_a[s % kWsAStages]);
                }
            }
        }
        cp_async_wait<0>();
        grid_dependency_wait();  // y, the scales and the workspace
        // ---------------- epilogue ----------------
        const bool got = (*abort_v == 0) && mbar_wait_ns(acc_full, 0, kWaitNs);
        if (!got) *abort_v = 1;
        tc_fence_after();
        // every decoder warp takes the same branch: abort is only set before
        // this point by a role that gave up, or just above by a lane whose
        // wait failed (then its warp-mates see it through the ballot)
        const bool warp_ok = __all_sync(0xffffffffu, got);
        if (warp_ok && dg == 0 && cluster_ks == 0 && tail_idx < 0) {
            const int q = warp & 3;  // TMEM lane quarter of this warp
            const int row = m0 + q * 32 + lane;
            const float sc = (row < L.out && scales) ? __half2float(__ushort_as_half(scales[row])) : 1.f;
            const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                float v[16];
                tmem_ld16(tbase + c0, v);
                const int gn = n0 + c0;
                if (row < L.out && gn < T) {
                    uint16_t *dst = y + (size_t)row * T + gn;
                    if (gn + 16 <= T) {
                        const uint4 o0 = make_uint4(f2h2(sc * v[0], sc * v[1]), f2h2(sc * v[2], sc * v[3]),
                                                    f2h2(sc * v[4], sc * v[5]), f2h2(sc * v[6], sc * v[7]));
                        const uint4 o1 = make_uint4(f2h2(sc * v[8], sc * v[9]), f2h2(sc * v[10], sc * v[11]),
                                                    f2h2(sc * v[12], sc * v[13]), f2h2(sc * v[14], sc * v[15]));
                        reinterpret_cast<uint4 *>(dst)[0] = o0;
                        reinterpret_cast<uint4 *>(dst)[1] = o1;
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (gn + j < T) dst[j] = __half_as_ushort(__float2half_rn(sc * v[j]));
                    }
                }
            }
        }
    }
    grid_dependency_wait();  // every thread, before the workspace and y
    __syncthreads();
    if (*abort_v) {
        // something gave up: record it and drain what was issued (bounded)
        if (tid == 0) record_status(ws, AQ_ERR_TIMEOUT);
        if (tid == 32) mbar_wait_ns(acc_full, 0, kWaitNs);
        if (tid == 0)
            for (int s = max(0, nk - kWsStages); s < nk; ++s)
                mbar_wait_ns(&full_b[s % kWsStages], (s / kWsStages) & 1, kWaitNs);
    }
    if (cluster_ks > 1) {
        // the decoder warps finish: warp & 3 is their TMEM lane quarter
        constexpr int NW = 4 * kWsGroupsOf<S>;
        gemm_cluster_finish<BN, NW>(L, tmem, sp.partials, m0, n0, T, cluster_ks, scales, y,
                                    warp >= 2 ? warp - 2 : -1, *abort_v == 0);
    }
    if (tail_idx >= 0) {
        // a tail tile's split: the last of its splits finishes it
        constexpr int NW = 4 * kWsGroupsOf<S>;
        float *slices = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) + kWsData) +
                        (size_t)tail_idx * tm.ks * kBM * BN;
        unsigned *counter = reinterpret_cast<unsigned *>(reinterpret_cast<char *>(ws) + kWsHeader) + tail_idx;
        gemm_tail_finish<BN, NW>(L, tmem, slices, counter, m0, n0, T, z, tm.ks, scales, y,
                                 warp >= 2 ? warp - 2 : -1, *abort_v == 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, BN);
}

// ---- self-test of the bounded wait -----------------------------------------

__global__ void selftest_wait_kernel(void *ws, int spin_limit)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival that never comes
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait_bounded(&bar, 0, (uint32_t)spin_limit)) record_status(ws, AQ_ERR_TIMEOUT);
    }
}

}  // namespace aqk

namespace aqh {
using namespace aqk;

// Launch plan of the TMA path (T % 8 == 0): token tile, split-K, workspace.
struct GemmPlan {
    bool tma;         // warp-specialised kernel (X by TMA)
    int bn;           // tokens per CTA: 512 above 256 tokens, else 256
    int mtiles, ntiles;
    int ks;           // splits of the input features (blockIdx.z)
    int per_split;    // 64-feature stages per split
    bool cluster;     // the splits form one cluster and finish on chip
    TailMap tail;     // ks > 0: the tail mode's 1-D grid
    size_t ws_bytes;  // status word + tile counters + fp32 partials
};

static GemmPlan plan_gemm(const Geom &g, int T)
{
    GemmPlan p{};
    p.tma = (T % 8) == 0;
    p.ws_bytes = kWsHeader;
    if (!p.tma) return p;
    p.mtiles = (g.out + kBM - 1) / kBM;
    // 512-token tiles halve the decode work per MMA; when they would leave
    // more than half the SMs without a tile (and so need a deep split of
    // the input features, whose partial sums cost a pass through L2),
    // 256-token tiles with fewer splits are faster (measured on Llama-2-7B
    // shapes at 512 tokens)
    // 512-token tiles halve the decode work per MMA; with few row tiles
    // (a 4096-row layer at 512 tokens) they need a split of the input
    // features, which the cluster finish makes cheap
    p.bn = T >= 384 || (T > 256 && (long)p.mtiles * ((T + 511) / 512) * 2 >= kNumSMs) ? 512 : 256;
    p.ntiles = (T + p.bn - 1) / p.bn;
    const int nst = (g.in + kBK - 1) / kBK;
    const long tiles = (long)p.mtiles * p.ntiles;
    // the decode is the bound: split the input features until about one CTA
    // per SM works, keeping at least 8 stages per split
    int ks = tiles < kNumSMs ? (int)(kNumSMs / tiles) : 1;
    ks = std::max(1, std::min(ks, nst / 8));
    // the split runs as one thread-block cluster along z whose CTAs share
    // the finish: 2, 4 or 8 CTAs (the largest power of two not above ks).
    // With at least 8 stages per split (nst >= 8 kc) none of them is empty:
    // per = ceil(nst / kc) gives exactly kc non-empty splits
    if (ks >= 2) {
        int kc = 2;
        while (kc * 2 <= std::min(ks, 8)) kc *= 2;
        ks = kc;
    }
    p.per_split = (nst + ks - 1) / ks;
    p.ks = (nst + p.per_split - 1) / p.per_split;
    p.cluster = p.ks > 1;
    if (p.ks > 1) p.ws_bytes = kWsData + (size_t)p.ks * tiles * kBM * p.bn * sizeof(float);
    // more tiles than one wave, the last wave at most half full: its tiles'
    // input features are split so that it fills the SMs (Llama-2-7B MLP
    // rows at 2048 tokens: 344 tiles, 48 in the third wave, split 3 ways)
    if (p.ks == 1 && tiles > kNumSMs) {
        const long tail = tiles % kNumSMs;
        if (tail > 0 && tail * 2 <= kNumSMs && tail <= kWsMaxCounters) {
            int kt = std::min((int)(kNumSMs / tail), std::min(nst / 8, 8));
            if (kt >= 2) {
                const int per = (nst + kt - 1) / kt;
                kt = (nst + per - 1) / per;  // no empty split
                p.tail = TailMap{(int)(tiles - tail), kt, per};
                p.ws_bytes = kWsData + (size_t)tail * kt * kBM * p.bn * sizeof(float);
            }
        }
    }
    return p;
}

size_t gemm_workspace_bytes(const Geom &g, int T) { return plan_gemm(g, T).ws_bytes; }

template <class S>
static constexpr int gemm_smem_bytes()
{
    return 1024 /* alignment slack */ + kStages * (kTileABytes + kTileBBytes) + S::kSmemBookBytes +
           kStages * 8 + 16;
}

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

template <class S, int BN>
static constexpr int gemm_ws_smem_bytes()
{
    return 1024 + kWsAStagesOf<S, BN> * kTileABytes + kWsStagesOf<S, BN> * (kBK * BN * 2) + S::kSmemBookBytes +
           (2 * kWsAStagesOf<S, BN> + 2 * kWsStagesOf<S, BN> + 1) * 8 + 16;
}

cudaError_t launch_gemm(const Geom &g, const void *packed, const uint16_t *cb,
                        const uint16_t *scales, const uint16_t *x, int T, uint16_t *y, void *ws,
                        cudaStream_t s, bool pdl)
{
    const uint8_t *pk = reinterpret_cast<const uint8_t *>(packed);
    const uint4 *c = reinterpret_cast<const uint4 *>(cb);
    const GemmPlan p = plan_gemm(g, T);
    PFN_cuTensorMapEncodeTiled_v12000 encode = p.tma ? tensor_map_encoder() : nullptr;
    if (encode) {
        // X [in][T] binary16: innermost dimension tokens, box 64 tokens x 64 features
        CUtensorMap map;
        cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)g.in};
        cuuint64_t strides[1] = {(cuuint64_t)T * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)kBK};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(x), dims, strides,
                            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        const long tiles = (long)p.mtiles * p.ntiles;
        const dim3 grid = p.tail.ks > 0 ? dim3((unsigned)(p.tail.full + (tiles - p.tail.full) * p.tail.ks), 1, 1)
                                        : dim3(p.mtiles, p.ntiles, p.ks);
        GemmSplit sp{nullptr};
        if (p.ks > 1) sp.partials = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) + kWsData);
        auto launch = [&](auto sch, auto bn) {
            using S = decltype(sch);
            constexpr int BN = decltype(bn)::value;
            constexpr int smem = gemm_ws_smem_bytes<S, BN>();
            static_assert(smem <= 227 * 1024, "shared memory of the warp-specialised GEMM");
            cudaError_t e = cudaFuncSetAttribute(gemm_ws_kernel<S, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem);
            if (e != cudaSuccess) return e;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = grid;
            cfg.blockDim = dim3(kWsThreadsOf<S>);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = s;
            cudaLaunchAttribute attr[2];
            int na = 0;
            if (p.cluster) {
                attr[na].id = cudaLaunchAttributeClusterDimension;
                attr[na].val.clusterDim.x = 1;
                attr[na].val.clusterDim.y = 1;
                attr[na].val.clusterDim.z = p.ks;
                ++na;
            }
            if (pdl) {
                attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                attr[na].val.programmaticStreamSerializationAllowed = 1;
                ++na;
            }
            cfg.attrs = attr;
            cfg.numAttrs = na;
            e = cudaLaunchKernelEx(&cfg, gemm_ws_kernel<S, BN>, map, g, pk, c, scales, T, y, ws, sp, p.per_split,
                                   p.cluster ? p.ks : 0, p.tail);
            if (e != cudaSuccess) return e;
            return cudaGetLastError();
        };
        return with_scheme(g, [&](auto sch) {
            return p.bn == 512 ? launch(sch, std::integral_constant<int, 512>{})
                               : launch(sch, std::integral_constant<int, 256>{});
        });
    }
    // T not a multiple of 8: rows of X are not 16-byte aligned for TMA; the
    // two-stage kernel stages X with ordinary loads.
    const dim3 grid((g.out + kBM - 1) / kBM, (T + kBN - 1) / kBN);
    return with_scheme(g, [&](auto sch) {
        using S = decltype(sch);
        constexpr int smem = gemm_smem_bytes<S>();
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        gemm_tc_kernel<S><<<grid, kGemmThreads, smem, s>>>(g, pk, c, scales, x, T, y, ws);
        return cudaGetLastError();
    });
}

cudaError_t launch_selftest_wait(void *ws, int spin_limit, cudaStream_t s)
{
    selftest_wait_kernel<<<1, 32, 0, s>>>(ws, spin_limit);
    return cudaGetLastError();
}

}  // namespace aqh
