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
#include "aq_common.cuh"

namespace aqk {

constexpr int kBM = 128;           // rows of W per CTA (MMA M)
constexpr int kBN = 128;           // tokens per CTA (MMA N)
constexpr int kBK = 64;            // input features per stage (8 groups)
constexpr int kStages = 2;
constexpr int kGemmThreads = 128;  // 4 warps: decode, stage X, epilogue
constexpr int kTileABytes = kBM * kBK * 2;  // 16 KiB
constexpr int kTileBBytes = kBK * kBN * 2;  // 16 KiB
constexpr uint64_t kWaitNs = 1000000000ull; // 1 s per wait

// ---- PTX wrappers -----------------------------------------------------------

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for a phase of an mbarrier for at most `ns` nanoseconds.
__device__ __forceinline__ bool mbar_wait_ns(uint64_t *bar, uint32_t parity, uint64_t ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 0; i < (1u << 30); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > ns) return false;
    }
    return false;
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; accumulate selects D += vs D =.
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Arrive (once) on `bar` when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 16 consecutive fp32 columns of tensor memory -> 16 registers.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float v[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor (sm_100 layout): start address >> 4 in
// bits 0-13, leading byte offset >> 4 in 16-29, stride byte offset >> 4 in
// 32-45, descriptor version 1 in bits 46-47, swizzle mode in 61-63
// (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3fff);
    d |= (uint64_t)((lbo >> 4) & 0x3fff) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fff) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor for kind::f16: fp32 accumulator (bits 4-5 = 1),
// binary16 A and B (formats 0), A K-major (bit 15 = 0), B MN-major
// (bit 16 = 1), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N)
{
    return (1u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | (1u << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled
// tile of 128-byte rows (rows 8-aligned into 1024-byte atoms).
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t c)
{
    return row * 128u + ((c ^ (row & 7u)) << 4);
}

// ---- kernel -----------------------------------------------------------------

template <int K>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(Geom L, const uint4 *__restrict__ packed, const uint4 *__restrict__ cb,
               const uint16_t *__restrict__ scales, const uint16_t *__restrict__ x, int T,
               uint16_t *__restrict__ y, void *ws)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
    uint8_t *smem = smem_raw + pad;
    uint8_t *tileA = smem;                                // [2][16 KiB]
    uint8_t *tileB = smem + kStages * kTileABytes;        // [2][16 KiB]
    uint4 *scb = reinterpret_cast<uint4 *>(tileB + kStages * kTileBBytes);  // 2x8 codebooks
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(scb) + 512 * 16);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kStages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * kBM;
    const int n0 = blockIdx.y * kBN;

    if (K == 2)
        for (int i = tid; i < 512; i += kGemmThreads) scb[i] = cb[i];
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
            uint32_t wd[8];
            const bool live = (rt < L.rtiles) && (g < L.G);
            if (live) {
                uint4 c = ldg_nc_v4(packed + (size_t)rt * L.gp + g);
                wd[0] = c.x & 0xffff; wd[1] = c.x >> 16; wd[2] = c.y & 0xffff; wd[3] = c.y >> 16;
                wd[4] = c.z & 0xffff; wd[5] = c.z >> 16; wd[6] = c.w & 0xffff; wd[7] = c.w >> 16;
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (live) {
                    if (K == 1)
                        v = ldg_nc_v4(cb + wd[r]);
                    else
                        v = add_round_h8(scb[wd[r] & 0xff], scb[256 + (wd[r] >> 8)]);
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

size_t gemm_workspace_bytes(const Geom &, int) { return kWsHeader; }

static constexpr int gemm_smem_bytes()
{
    return 1024 /* alignment slack */ + kStages * (kTileABytes + kTileBBytes) + 512 * 16 +
           kStages * 8 + 16;
}

cudaError_t launch_gemm(const Geom &g, const void *packed, const uint16_t *cb,
                        const uint16_t *scales, const uint16_t *x, int T, uint16_t *y, void *ws,
                        cudaStream_t s)
{
    const int smem = gemm_smem_bytes();
    dim3 grid((g.out + kBM - 1) / kBM, (T + kBN - 1) / kBN);
    const uint4 *pk = reinterpret_cast<const uint4 *>(packed);
    const uint4 *c = reinterpret_cast<const uint4 *>(cb);
    cudaError_t e;
    if (g.K == 1) {
        e = cudaFuncSetAttribute(gemm_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        gemm_tc_kernel<1><<<grid, kGemmThreads, smem, s>>>(g, pk, c, scales, x, T, y, ws);
    } else {
        e = cudaFuncSetAttribute(gemm_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        gemm_tc_kernel<2><<<grid, kGemmThreads, smem, s>>>(g, pk, c, scales, x, T, y, ws);
    }
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(void *ws, int spin_limit, cudaStream_t s)
{
    selftest_wait_kernel<<<1, 32, 0, s>>>(ws, spin_limit);
    return cudaGetLastError();
}

}  // namespace aqh
