// Gradient of L = sum(gy * y), y = diag(s) W x, with respect to the row
// scales and the codebooks (sm_100a).
//
// The codebooks are learned jointly with the codes by minimising the
// layer's output error (AQLM wiki entry, "Niveau tech avancé"); the step
// that fine-tunes them needs, with the decode's binary16 rounding taken as
// the identity,
//     M[o][i]         = sum_b gy[o][b] x[i][b]                 (a dense GEMM)
//     grad_s[o]       = sum_i W[o][i] M[o][i]
//     grad_C[k][c][j] = sum of s[o] M[o][8g+j] over the (o, g) whose code k is c.
//
// One persistent kernel (a CTA per SM walks 128-row x 128-feature tiles,
// 16 groups each, with two accumulator buffers in tensor memory so the
// epilogue of one tile overlaps the MMAs of the next); the
// contraction over tokens runs on the tensor cores (tcgen05.mma kind::f16,
// both operands K-major, 128-byte swizzle, loaded by TMA without multicast,
// fp32 accumulator in tensor memory).  The epilogue reads M from TMEM, one
// row per thread: it decodes the row's 16 weight groups for grad_s, and
// scatters s[o] M into grad_C.  8-bit codebooks: fp32 accumulators in shared
// memory, one private copy per epilogue warp, updated without atomics (lanes
// holding the same codeword take turns, found with __match_any_sync; shared
// float atomics cost 2.5x the whole kernel here), summed and flushed to
// global memory once per CTA; 8x8, whose four copies would not fit, keeps
// one copy with shared atomics.  16-bit codebooks (65536 entries): global
// float4 atomics.  Global atomics make the summation order of grad_C and
// grad_s vary from run to run (fp32 rounding only).
//
// Roles: warp 0 TMA producer, warp 1 MMA issuer, warps 2-5 epilogue.  Every
// wait is bounded; on give-up the kernel records AQ_ERR_TIMEOUT, drains what
// it issued (bounded), frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "scheme.cuh"
#include "tc_common.cuh"

namespace aqk {

constexpr int kGradBM = 128;                      // rows of W per CTA (MMA M)
constexpr int kGradBN = 128;                      // input features per CTA (MMA N)
constexpr int kGradBK = 64;                       // tokens per stage
constexpr int kGradThreads = 192;                 // 6 warps
constexpr int kGradEpilogueThreads = 128;         // warps 2-5
constexpr int kGradTileA = kGradBM * kGradBK * 2;  // 16 KiB of gy
constexpr int kGradTileB = kGradBN * kGradBK * 2;  // 16 KiB of x

// Ring depth: 4 stages; 3 when 8-bit codebooks and their fp32 gradient
// accumulators take K x 12 KiB of shared memory with K = 8.
template <class S>
constexpr int kGradStagesOf = (S::kSmemBookBytes > 8192) ? 3 : 4;

// 8-bit codebook gradients accumulate in shared memory: one private copy
// per epilogue warp (race-free adds, no atomics) when four copies fit, else
// (8x8) one copy updated with shared-memory atomics.
template <class S>
constexpr bool kGradPrivateAcc = S::kBooksInSmem && S::K <= 2;

template <class S>
constexpr int grad_acc_floats()
{
    return S::kBooksInSmem ? S::K * 256 * 8 * (kGradPrivateAcc<S> ? 4 : 1) : 0;
}

template <class S>
constexpr int grad_smem_bytes()
{
    return 1024 + kGradStagesOf<S> * (kGradTileA + kGradTileB) + S::kSmemBookBytes + grad_acc_floats<S>() * 4 +
           (2 * kGradStagesOf<S> + 4) * 8 + 16;
}

// The packed word of (row o, group g): K*B/8 bytes.
template <class S>
__device__ __forceinline__ uint64_t load_word(const Geom &L, const uint8_t *__restrict__ packed, int o, int g)
{
    const uint8_t *p = packed + ((size_t)(o >> 3) * L.gp + g) * S::kChunkBytes + (size_t)(o & 7) * S::kWordBytes;
    if constexpr (S::kWordBytes == 1) return *p;
    else if constexpr (S::kWordBytes == 2) return *reinterpret_cast<const uint16_t *>(p);
    else if constexpr (S::kWordBytes == 4) return *reinterpret_cast<const uint32_t *>(p);
    else return *reinterpret_cast<const uint64_t *>(p);
}

template <class S>
__global__ void __launch_bounds__(kGradThreads, 1)
param_grad_kernel(const __grid_constant__ CUtensorMap gymap, const __grid_constant__ CUtensorMap xmap, Geom L,
                  const uint8_t *__restrict__ packed, const uint4 *__restrict__ cb,
                  const uint16_t *__restrict__ scales, int T, float *__restrict__ grad_s,
                  float *__restrict__ grad_cb, void *ws)
{
    constexpr int ST = kGradStagesOf<S>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *tileA = smem;                                        // [ST][16 KiB] gy
    uint8_t *tileB = tileA + ST * kGradTileA;                     // [ST][16 KiB] x
    uint4 *scb = reinterpret_cast<uint4 *>(tileB + ST * kGradTileB);  // B = 8 codebooks
    float *sacc = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(scb) + S::kSmemBookBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(sacc + grad_acc_floats<S>());
    uint64_t *empty = full + ST;
    uint64_t *acc_full = empty + ST;   // [2] accumulator buffer ready for the epilogue
    uint64_t *acc_empty = acc_full + 2;  // [2] accumulator buffer drained by the epilogue
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    uint32_t *abort_flag = tmem_slot + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntn = (L.in + kGradBN - 1) / kGradBN;
    const int ntiles = ((L.out + kGradBM - 1) / kGradBM) * ntn;
    const int nk = (T + kGradBK - 1) / kGradBK;

    if constexpr (S::kBooksInSmem) {
        for (int i = tid; i < S::K * 256; i += kGradThreads) scb[i] = cb[i];
        for (int i = tid; i < grad_acc_floats<S>(); i += kGradThreads) sacc[i] = 0.f;
    }
    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kGradEpilogueThreads);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 2 * kGradBN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile uint32_t *abort_v = abort_flag;

    // This CTA's tiles: t = blockIdx.x + gridDim.x * lt, row block t / ntn,
    // feature block t % ntn.  Stage counter q runs across tiles.
    if (warp == 0) {
        // ---------------- TMA producer: gy and x tiles ----------------
        if (lane == 0) {
            int q = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort_v; t += gridDim.x) {
                const int m0 = (t / ntn) * kGradBM, n0 = (t % ntn) * kGradBN;
                for (int s = 0; s < nk; ++s, ++q) {
                    const int buf = q % ST;
                    if (q >= ST && !mbar_wait_ns(&empty[buf], ((q / ST) - 1) & 1, kWaitNs)) {
                        *abort_v = 1;
                        break;
                    }
                    if (*abort_v) break;
                    mbar_arrive_expect_tx(&full[buf], kGradTileA + kGradTileB);
                    tma_load_2d(smem_u32(tileA + buf * kGradTileA), &gymap, s * kGradBK, m0, &full[buf]);
                    tma_load_2d(smem_u32(tileB + buf * kGradTileB), &xmap, s * kGradBK, n0, &full[buf]);
                }
            }
            // copies of the last ring's worth of stages may still be landing
            // (only after an abort): wait for them, bounded
            for (int qq = max(0, q - ST); qq < q; ++qq) mbar_wait_ns(&full[qq % ST], (qq / ST) & 1, kWaitNs);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = make_idesc(kGradBM, kGradBN, false);  // both operands K-major
            int q = 0, lt = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort_v; t += gridDim.x, ++lt) {
                const int ab = lt & 1;
                // the epilogue has drained this accumulator buffer (tile lt - 2)
                if (lt >= 2 && !mbar_wait_ns(&acc_empty[ab], ((lt >> 1) - 1) & 1, kWaitNs)) {
                    *abort_v = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(ab * kGradBN);
                for (int s = 0; s < nk; ++s, ++q) {
                    const int buf = q % ST;
                    if (!mbar_wait_ns(&full[buf], (q / ST) & 1, kWaitNs)) {
                        *abort_v = 1;
                        break;
                    }
                    if (*abort_v) break;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(tileA + buf * kGradTileA);
                    const uint32_t b0 = smem_u32(tileB + buf * kGradTileB);
#pragma unroll
                    for (int ks = 0; ks < kGradBK / 16; ++ks) {
                        const uint64_t ad = smem_desc_sw128(a0 + ks * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(b0 + ks * 32, 16, 1024);
                        mma_f16_ss(acc, ad, bd, idesc, (s > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(&empty[buf]);
                }
                mma_commit(&acc_full[ab]);  // completes when this tile's MMAs have
            }
            // the last stage's commit completes once every MMA issued here has:
            // none may still write tensor memory when it is freed
            if (q > 0) mbar_wait_ns(&empty[(q - 1) % ST], ((q - 1) / ST) & 1, kWaitNs);
        }
    } else {
        // ---------------- epilogue: one row per thread, tile after tile ----------------
        const int qd = warp & 3;  // TMEM lane quarter of this warp
        float *wacc = sacc + (kGradPrivateAcc<S> ? (warp - 2) * S::K * 256 * 8 : 0);
        int lt = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
            const int ab = lt & 1;
            const int m0 = (t / ntn) * kGradBM, n0 = (t % ntn) * kGradBN;
            const int o = m0 + qd * 32 + lane;
            const bool row_ok = o < L.out;
            // 8-bit codebooks with private accumulators: this row's codes of
            // the tile's 16 groups are requested before the accumulator is
            // waited for (they do not depend on it), so the scatter rounds of
            // the slices below do not each wait on an L2 round trip; the
            // other schemes read them slice by slice (measured faster there)
            constexpr bool kPrefetch = kGradPrivateAcc<S>;
            uint64_t words[kGradBN / 8];
            if constexpr (kPrefetch) {
#pragma unroll
                for (int q = 0; q < kGradBN / 8; ++q) {
                    const int g = n0 / 8 + q;
                    words[q] = (row_ok && g < L.G) ? load_word<S>(L, packed, o, g) : 0ull;
                }
            }
            const bool got = (*abort_v == 0) && mbar_wait_ns(&acc_full[ab], (lt >> 1) & 1, kWaitNs);
            if (!got) *abort_v = 1;
            // tcgen05.ld is warp-collective: a failed wait in any lane ends the warp
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const float so = (row_ok && scales) ? __half2float(__ushort_as_half(scales[o])) : 1.f;
            const uint32_t tbase = tmem + (uint32_t)(ab * kGradBN) + ((uint32_t)(qd * 32) << 16);
            float gs = 0.f;
            auto slice = [&](int c0) {
                float v[16];
                tmem_ld16(tbase + c0, v);  // M[o][n0 + c0 .. + 15]: two groups
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int g = (n0 + c0) / 8 + h;
                    if (g >= L.G) continue;  // the same for the whole warp
                    uint32_t code[S::K];
                    uint64_t word = 0;
                    if constexpr (kPrefetch) word = words[c0 / 8 + h];
                    else if (row_ok) word = load_word<S>(L, packed, o, g);
#pragma unroll
                    for (int k = 0; k < S::K; ++k) code[k] = (uint32_t)(word >> (k * S::B)) & S::kMask;
                    const float *m = v + 8 * h;
                    if (grad_s && row_ok) {
                        uint4 t[S::K];
#pragma unroll
                        for (int k = 0; k < S::K; ++k) {
                            if constexpr (S::kBooksInSmem)
                                t[k] = scb[k * 256 + code[k]];
                            else
                                t[k] = ldg_nc_v4(cb + ((size_t)k << S::B) + code[k]);
                        }
                        const uint4 wv = sum_round_fast_h8<S::K>(t);
                        const float2 w0 = h2f2(wv.x), w1 = h2f2(wv.y), w2 = h2f2(wv.z), w3 = h2f2(wv.w);
                        gs = fmaf(w0.x, m[0], gs); gs = fmaf(w0.y, m[1], gs);
                        gs = fmaf(w1.x, m[2], gs); gs = fmaf(w1.y, m[3], gs);
                        gs = fmaf(w2.x, m[4], gs); gs = fmaf(w2.y, m[5], gs);
                        gs = fmaf(w3.x, m[6], gs); gs = fmaf(w3.y, m[7], gs);
                    }
                    if (grad_cb) {
#pragma unroll
                        for (int k = 0; k < S::K; ++k) {
                            const float4 a0 = make_float4(so * m[0], so * m[1], so * m[2], so * m[3]);
                            const float4 a1 = make_float4(so * m[4], so * m[5], so * m[6], so * m[7]);
                            if constexpr (kGradPrivateAcc<S>) {
                                // lanes with the same codeword take turns (rank among
                                // their peers); other lanes' rows go in the same round
                                const uint32_t key = row_ok ? (uint32_t)code[k] : 0x10000u + lane;
                                const uint32_t peers = __match_any_sync(0xffffffffu, key);
                                const int rank = __popc(peers & ((1u << lane) - 1u));
                                const int rounds = (int)__reduce_max_sync(0xffffffffu, (uint32_t)__popc(peers));
                                float4 *dst = reinterpret_cast<float4 *>(wacc + (k * 256 + code[k]) * 8);
                                for (int r = 0; r < rounds; ++r) {
                                    if (row_ok && rank == r) {
                                        float4 b0 = dst[0], b1 = dst[1];
                                        b0.x += a0.x; b0.y += a0.y; b0.z += a0.z; b0.w += a0.w;
                                        b1.x += a1.x; b1.y += a1.y; b1.z += a1.z; b1.w += a1.w;
                                        dst[0] = b0;
                                        dst[1] = b1;
                                    }
                                    __syncwarp();
                                }
                            } else if constexpr (S::kBooksInSmem) {
                                if (row_ok) {
                                    float *a = wacc + (k * 256 + code[k]) * 8;
#pragma unroll
                                    for (int j = 0; j < 8; ++j) atomicAdd(a + j, so * m[j]);
                                }
                            } else if (row_ok) {
                                float4 *a = reinterpret_cast<float4 *>(grad_cb + (((size_t)k << S::B) + code[k]) * 8);
                                atomicAdd(a, a0);
                                atomicAdd(a + 1, a1);
                            }
                        }
                    }
                }
            };
            if constexpr (kPrefetch) {
#pragma unroll
                for (int c0 = 0; c0 < kGradBN; c0 += 16) slice(c0);
            } else {
#pragma unroll 1
                for (int c0 = 0; c0 < kGradBN; c0 += 16) slice(c0);
            }
            if (row_ok && grad_s) atomicAdd(grad_s + o, gs);
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);  // this thread is done with the buffer
        }
    }
    __syncthreads();
    if (*abort_v) {
        if (tid == 0) record_status(ws, AQ_ERR_TIMEOUT);
    } else if constexpr (S::kBooksInSmem) {
        // this CTA's share of the 8-bit codebook gradient, once
        if (grad_cb) {
            constexpr int n4 = S::K * 256 * 8 / 4;  // float4 per copy
            constexpr int copies = kGradPrivateAcc<S> ? 4 : 1;
            const float4 *acc4 = reinterpret_cast<const float4 *>(sacc);
            for (int i = tid; i < n4; i += kGradThreads) {
                float4 a = acc4[i];
#pragma unroll
                for (int w = 1; w < copies; ++w) {
                    const float4 b = acc4[w * n4 + i];
                    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                }
                if (a.x != 0.f || a.y != 0.f || a.z != 0.f || a.w != 0.f)
                    atomicAdd(reinterpret_cast<float4 *>(grad_cb) + i, a);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 2 * kGradBN);
}

}  // namespace aqk

namespace aqh {
using namespace aqk;

size_t param_grad_workspace_bytes(const Geom &, int) { return kWsHeader; }

static PFN_cuTensorMapEncodeTiled_v12000 grad_tensor_map_encoder()
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

// [rows][T] binary16, tokens innermost: boxes of 64 tokens x 128 rows, 128-byte swizzle.
static bool token_major_map(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *map, const uint16_t *base,
                            int rows, int T)
{
    cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)T * 2};
    cuuint32_t box[2] = {(cuuint32_t)kGradBK, 128};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_param_grad(const Geom &g, const void *packed, const uint16_t *cb, const uint16_t *scales,
                              const uint16_t *x, const uint16_t *gy, int T, float *grad_s, float *grad_cb,
                              void *ws, cudaStream_t s)
{
    // outputs are overwritten: the kernel adds into zeroed buffers
    if (grad_s) {
        cudaError_t e = cudaMemsetAsync(grad_s, 0, sizeof(float) * (size_t)g.out, s);
        if (e != cudaSuccess) return e;
    }
    if (grad_cb) {
        cudaError_t e = cudaMemsetAsync(grad_cb, 0, sizeof(float) * ((size_t)g.K << g.B) * 8, s);
        if (e != cudaSuccess) return e;
    }
    if (!grad_s && !grad_cb) return cudaSuccess;
    PFN_cuTensorMapEncodeTiled_v12000 encode = grad_tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap gymap, xmap;
    if (!token_major_map(encode, &gymap, gy, g.out, T) || !token_major_map(encode, &xmap, x, g.in, T))
        return cudaErrorInvalidValue;
    // persistent: one CTA per SM (its shared memory allows no second), each
    // walking tiles blockIdx.x, blockIdx.x + gridDim.x, ...
    const long ntiles = (long)((g.out + kGradBM - 1) / kGradBM) * ((g.in + kGradBN - 1) / kGradBN);
    const dim3 grid((unsigned)std::min<long>(ntiles, kNumSMs));
    const uint8_t *pk = reinterpret_cast<const uint8_t *>(packed);
    const uint4 *c = reinterpret_cast<const uint4 *>(cb);
    return with_scheme(g, [&](auto sch) {
        using S = decltype(sch);
        constexpr int smem = grad_smem_bytes<S>();
        static_assert(smem <= 227 * 1024, "shared memory of the gradient kernel");
        cudaError_t e = cudaFuncSetAttribute(param_grad_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        param_grad_kernel<S><<<grid, kGradThreads, smem, s>>>(gymap, xmap, g, pk, c, scales, T, grad_s, grad_cb, ws);
        return cudaGetLastError();
    });
}

}  // namespace aqh
