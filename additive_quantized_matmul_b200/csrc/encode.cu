// Encoder: beam search of the codes of a layer for fixed 8-bit codebooks
// (1x8, 2x8, 8x8) under the quantisation objective of "Extreme Compression
// of Large Language Models via Additive Quantization" (AQLM wiki entry,
// "Niveau tech avancé"): || W - sum_k C_k[i_k] ||^2_H with H = 2 X^T X, the
// codes assigned by beam search.  The objective is a sum over output rows of
// e^T H e (e = w - reconstruction), so rows are independent: one CTA per row.
//
// Per row, groups in order, the others fixed: for group g the beam runs over
// the group's K codes, codebook by codebook; every beam proposes each of the
// 256 codes for slot (g, k); the `beam` proposals with the smallest
// objective survive, ordered by (objective, parent beam, code); the best
// beam is committed before group g + 1.  With the group's reconstruction
// changed by D (8 values), the objective changes by
//     delta = -2 D^T v + D^T H_gg D,   v = (H e)_g, H_gg the diagonal block,
// and for a proposal D = a_b + C_k[c] (a_b = the beam's change so far minus
// the slot's starting codeword) this is
//     delta = const_b + q_gk(c) + 2 C_k[c] . w_b,
//     const_b = a_b^T H_gg a_b - 2 a_b^T v,  w_b = H_gg a_b - v,
//     q_gk(c) = C_k[c]^T H_gg C_k[c]           (a per-layer table).
// The group's objective before the change is common to all its proposals,
// so ranking by delta ranks by the objective.  fp32 throughout (exact for
// integer-valued inputs of moderate size, which the tests use).
#include <cuda_fp16.h>

#include <type_traits>

#include "scheme.cuh"

namespace aqk {

constexpr int kEncThreads = 256;   // one per code of an 8-bit codebook
constexpr int kEncMaxBeam = 16;

// q[(g * K + k) * 256 + c] = C_k[c]^T H_gg C_k[c]
template <int K>
__global__ void __launch_bounds__(256) encode_q_kernel(int in, const float *__restrict__ h,
                                                       const uint4 *__restrict__ cb, float *__restrict__ q)
{
    __shared__ float hgg[64];
    const int g = blockIdx.x, c = threadIdx.x;
    if (c < 64) hgg[c] = h[(size_t)(8 * g + c / 8) * in + 8 * g + c % 8];
    __syncthreads();
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
        const uint4 w = cb[k * 256 + c];
        const float2 a = h2f2(w.x), b = h2f2(w.y), d = h2f2(w.z), e = h2f2(w.w);
        const float x[8] = {a.x, a.y, b.x, b.y, d.x, d.y, e.x, e.y};
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float t = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) t = fmaf(hgg[i * 8 + j], x[j], t);
            acc = fmaf(x[i], t, acc);
        }
        q[((size_t)g * K + k) * 256 + c] = acc;
    }
}

__device__ __forceinline__ uint64_t enc_key(float s, int beam, int code)
{
    s = s + 0.f;  // -0 -> +0: equal objectives compare equal
    uint32_t u = __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // order-preserving
    return ((uint64_t)u << 32) | ((uint32_t)beam << 8) | (uint32_t)code;
}

__device__ __forceinline__ float key_score(uint64_t key)
{
    uint32_t u = (uint32_t)(key >> 32);
    u = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
    return __uint_as_float(u);
}

__device__ __forceinline__ uint64_t warp_min_u64(uint64_t v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t t = __shfl_xor_sync(0xffffffffu, v, o);
        v = t < v ? t : v;
    }
    return v;
}

__device__ __forceinline__ void load_f8(const uint4 w, float x[8])
{
    const float2 a = h2f2(w.x), b = h2f2(w.y), d = h2f2(w.z), e = h2f2(w.w);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y; x[4] = d.x; x[5] = d.y; x[6] = e.x; x[7] = e.y;
}

// Sorting network: the 16 keys of a thread in ascending order.
__device__ __forceinline__ void sort16(uint64_t (&k)[kEncMaxBeam])
{
#pragma unroll
    for (int pass = 0; pass < kEncMaxBeam; ++pass)
#pragma unroll
        for (int i = pass & 1; i + 1 < kEncMaxBeam; i += 2) {
            const uint64_t a = k[i], b = k[i + 1];
            k[i] = a < b ? a : b;
            k[i + 1] = a < b ? b : a;
        }
}

__device__ __forceinline__ void pop16(uint64_t (&k)[kEncMaxBeam])
{
#pragma unroll
    for (int i = 0; i + 1 < kEncMaxBeam; ++i) k[i] = k[i + 1];
    k[kEncMaxBeam - 1] = ~0ull;
}

template <int K>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(Geom L, const uint16_t *__restrict__ w,
                                                             const float *__restrict__ h, const uint4 *__restrict__ cb,
                                                             const float *__restrict__ qtab,
                                                             const uint8_t *__restrict__ codes_in,
                                                             uint8_t *__restrict__ codes_out, int beam)
{
    extern __shared__ float e[];                   // [in] residual w - reconstruction of this row
    __shared__ uint4 scb[K * 256];                 // the codebooks
    __shared__ float hgg[64], v[8];                // H_gg and (H e)_g of the current group
    __shared__ float bD[2][kEncMaxBeam][8];        // each beam's change of the group's reconstruction
    __shared__ uint8_t bcode[2][kEncMaxBeam][K];   // each beam's codes for the group
    __shared__ float bconst[kEncMaxBeam], bw[kEncMaxBeam][8];
    __shared__ uint64_t wtop[kEncThreads / 32][kEncMaxBeam];
    __shared__ uint64_t sel[kEncMaxBeam];
    const int o = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int in = L.in, G = L.G;
    const uint8_t *ci = codes_in + (size_t)o * G * K;
    const __half *cbh = reinterpret_cast<const __half *>(scb);

    for (int i = tid; i < K * 256; i += kEncThreads) scb[i] = cb[i];
    __syncthreads();
    for (int i = tid; i < in; i += kEncThreads) {
        const int g = i >> 3, j = i & 7;
        float r = 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k) r += __half2float(cbh[(k * 256 + ci[g * K + k]) * 8 + j]);
        e[i] = __half2float(__ushort_as_half(w[(size_t)o * in + i])) - r;
    }
    int cur = 0;
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
        __syncthreads();  // e holds every committed group
        {
            // v_j = sum_t H[8g + j][t] e[t], one warp per j (H rows coalesced)
            // eight independent loads in flight per lane (an L2 round trip
            // per step otherwise)
            const float *hr = h + (size_t)(8 * g + warp) * in;
            float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            int t = lane;
            for (; t + 7 * 32 < in; t += 8 * 32) {
                float hv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) hv[u] = __ldg(hr + t + 32 * u);
#pragma unroll
                for (int u = 0; u < 8; ++u) a8[u] = fmaf(hv[u], e[t + 32 * u], a8[u]);
            }
            for (; t < in; t += 32) a8[0] = fmaf(__ldg(hr + t), e[t], a8[0]);
            float acc = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) v[warp] = acc;
        }
        if (tid < 64) hgg[tid] = h[(size_t)(8 * g + tid / 8) * in + 8 * g + tid % 8];
        if (tid < 8) bD[cur][0][tid] = 0.f;
        if (tid < K) bcode[cur][0][tid] = ci[g * K + tid];
        int nb = 1;
        __syncthreads();
#pragma unroll 1
        for (int k = 0; k < K; ++k) {
            const uint32_t c0 = ci[g * K + k];  // the slot's starting code, common to all beams
            if (tid < nb) {
                float a[8], c0v[8], ha[8];
                load_f8(scb[k * 256 + c0], c0v);
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = bD[cur][tid][j] - c0v[j];
                float cst = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float t = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) t = fmaf(hgg[i * 8 + j], a[j], t);
                    ha[i] = t;
                    cst = fmaf(a[i], t - 2.f * v[i], cst);
                    bw[tid][i] = t - v[i];
                }
                bconst[tid] = cst;
            }
            __syncthreads();
            // scores of code c = tid for every beam
            uint64_t kk[kEncMaxBeam];
            {
                float x[8];
                load_f8(scb[k * 256 + tid], x);
                const float qc = qtab[((size_t)g * K + k) * 256 + tid];
#pragma unroll
                for (int b = 0; b < kEncMaxBeam; ++b) kk[b] = ~0ull;
#pragma unroll
                for (int b = 0; b < kEncMaxBeam; ++b) {
                    if (b >= nb) break;
                    float d = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) d = fmaf(x[i], bw[b][i], d);
                    kk[b] = enc_key(bconst[b] + qc + 2.f * d, b, tid);
                }
            }
            if (nb > 1) sort16(kk);  // one live beam: kk[0] is the only key
            // the warp's `beam` smallest keys (keys are unique)
            for (int r = 0; r < beam; ++r) {
                const uint64_t m = warp_min_u64(kk[0]);
                if (kk[0] == m) pop16(kk);
                if (lane == 0) wtop[warp][r] = m;
            }
            __syncthreads();
            if (warp == 0) {
                uint64_t hl[kEncMaxBeam];
#pragma unroll
                for (int i = 0; i < kEncMaxBeam; ++i)
                    hl[i] = (lane < kEncThreads / 32 && i < beam) ? wtop[lane][i] : ~0ull;
                for (int r = 0; r < beam; ++r) {
                    const uint64_t m = warp_min_u64(hl[0]);
                    if (hl[0] == m) pop16(hl);
                    if (lane == 0) sel[r] = m;
                }
            }
            __syncthreads();
            const int nxt = cur ^ 1;
            if (tid < beam) {
                const uint64_t key = sel[tid];
                const int pb = (int)((key >> 8) & 0xff), c = (int)(key & 0xff);
                float cv[8], c0v[8];
                load_f8(scb[k * 256 + c], cv);
                load_f8(scb[k * 256 + c0], c0v);
#pragma unroll
                for (int j = 0; j < 8; ++j) bD[nxt][tid][j] = bD[cur][pb][j] + cv[j] - c0v[j];
#pragma unroll
                for (int q = 0; q < K; ++q) bcode[nxt][tid][q] = bcode[cur][pb][q];
                bcode[nxt][tid][k] = (uint8_t)c;
            }
            nb = beam;
            cur = nxt;
            __syncthreads();
        }
        // commit the best beam of the group
        if (tid < 8) e[8 * g + tid] -= bD[cur][0][tid];
        if (tid < K) codes_out[((size_t)o * G + g) * K + tid] = bcode[cur][0][tid];
    }
}


// ---- 16-bit codebooks (1x16, 2x16) -----------------------------------------
// The same search over 65536 codes per slot.  One CTA per tile of kE16Rows
// rows (the codebook then streams through shared memory once per tile and
// slot instead of once per row); each row's codes are split over kE16Slices
// threads, each keeping its `nsel` best keys, merged per row at the slot's
// end.  The residual e lives in the workspace ([out][in] fp32), the table
// q[(g K + k) 65536 + c] = C_k[c]^T H_gg C_k[c] too.  Keys are (objective
// change, parent beam, code), as above, with 16-bit codes.  With K = 1 the
// one slot's best proposal is the group's (the beam keeps nothing past it);
// with K = 2 the first slot keeps `beam` proposals and the second its best.
constexpr int kE16Rows = 16;                     // rows per CTA
constexpr int kE16Slices = kEncThreads / kE16Rows;  // threads per row
constexpr int kE16Chunk = 512;                   // codes per shared-memory chunk
constexpr int kE16Cols = 256;                    // residual columns per chunk of (H e)_g
constexpr int encode16_smem_bytes()
{
    return kE16Rows * kE16Slices * kEncMaxBeam * 8 + kE16Chunk * 9 * 4 + kE16Rows * (kE16Cols + 1) * 4 +
           8 * kE16Cols * 4 + 2 * kE16Rows * kEncMaxBeam * 8 * 4 + kE16Rows * kEncMaxBeam * 8 * 4;
}

template <int K>
__global__ void __launch_bounds__(256) encode16_q_kernel(int in, const float *__restrict__ h,
                                                         const uint4 *__restrict__ cb, float *__restrict__ q)
{
    __shared__ float hgg[64];
    const int g = blockIdx.y;
    if (threadIdx.x < 64) hgg[threadIdx.x] = h[(size_t)(8 * g + threadIdx.x / 8) * in + 8 * g + threadIdx.x % 8];
    __syncthreads();
    const int c = blockIdx.x * 256 + threadIdx.x;  // code 0 .. 65535
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
        float x[8];
        load_f8(cb[(size_t)k * 65536 + c], x);
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float t = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) t = fmaf(hgg[i * 8 + j], x[j], t);
            acc = fmaf(x[i], t, acc);
        }
        q[((size_t)g * K + k) * 65536 + c] = acc;
    }
}

__device__ __forceinline__ uint64_t enc16_key(float s, int beam, int code)
{
    s = s + 0.f;  // -0 -> +0
    uint32_t u = __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | ((uint32_t)beam << 16) | (uint32_t)code;
}

template <int K>
__global__ void __launch_bounds__(kEncThreads) encode16_kernel(Geom L, const uint16_t *__restrict__ w,
                                                               const float *__restrict__ h,
                                                               const uint4 *__restrict__ cb,
                                                               const float *__restrict__ qtab,
                                                               const uint16_t *__restrict__ codes_in,
                                                               uint16_t *__restrict__ codes_out,
                                                               float *__restrict__ eg, int beam)
{
    constexpr int R = kE16Rows, S = kE16Slices;
    // dynamic shared memory (encode16_smem_bytes), carved:
    extern __shared__ __align__(16) uint8_t e16_smem[];
    auto lists = reinterpret_cast<uint64_t(*)[S][kEncMaxBeam]>(e16_smem);         // [R]: per-slice best keys
    auto sx = reinterpret_cast<float(*)[8]>(lists + R);                           // [kE16Chunk]: codebook chunk
    float *sq = reinterpret_cast<float *>(sx + kE16Chunk);                        // [kE16Chunk]: its q
    auto ec = reinterpret_cast<float(*)[kE16Cols + 1]>(sq + kE16Chunk);           // [R]: residual chunk
    auto hc = reinterpret_cast<float(*)[kE16Cols]>(ec + R);                       // [8]: H rows 8g.. chunk
    auto bD = reinterpret_cast<float(*)[R][kEncMaxBeam][8]>(hc + 8);              // [2]: beams' changes
    auto bw = reinterpret_cast<float(*)[kEncMaxBeam][8]>(bD + 2);                 // [R]: proposals' w
    __shared__ float hgg[64], v[R][8];
    __shared__ uint16_t bcode[2][R][kEncMaxBeam][K];
    __shared__ float bconst[R][kEncMaxBeam];
    __shared__ uint64_t sel[R][kEncMaxBeam];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // thread (row my_r, slice my_s): a warp's lanes are 16 rows x 2 slices,
    // so a codeword read serves 16 rows (2 codewords per warp access)
    static_assert(R == 16 && S == 16, "16 rows x 16 slices");
    const int my_r = lane & 15, my_s = (warp << 1) | (lane >> 4);
    const int in = L.in, G = L.G, o0 = blockIdx.x * R;
    const int nrows = min(R, L.out - o0);

    // e = w - the starting codes' reconstruction
    for (int i = tid; i < nrows * in; i += kEncThreads) {
        const int r = i / in, c = i - r * in, g = c >> 3, j = c & 7;
        const size_t o = (size_t)(o0 + r);
        float rec = 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            float x[8];
            load_f8(cb[(size_t)k * 65536 + codes_in[(o * G + g) * K + k]], x);
            rec += x[j];
        }
        eg[o * in + c] = __half2float(__ushort_as_half(w[o * in + c])) - rec;
    }
    int cur = 0;
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
        __syncthreads();  // e holds every committed group (global writes of this CTA)
        // v[r][j] = sum_t H[8g + j][t] e[r][t]: warp j, lane columns, 256-column chunks
        float acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < in; c0 += kE16Cols) {
            const int nc = min(kE16Cols, in - c0);
            for (int i = tid; i < R * kE16Cols; i += kEncThreads) {
                const int r = i / kE16Cols, c = i % kE16Cols;
                ec[r][c] = (r < nrows && c < nc) ? eg[(size_t)(o0 + r) * in + c0 + c] : 0.f;
            }
            for (int i = tid; i < 8 * kE16Cols; i += kEncThreads) {
                const int j = i / kE16Cols, c = i % kE16Cols;
                hc[j][c] = c < nc ? h[(size_t)(8 * g + j) * in + c0 + c] : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int m = 0; m < kE16Cols / 32; ++m) {
                const float hv = hc[warp][lane + 32 * m];
#pragma unroll
                for (int r = 0; r < R; ++r) acc[r] = fmaf(hv, ec[r][lane + 32 * m], acc[r]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float a = acc[r];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
            if (lane == 0) v[r][warp] = a;
        }
        if (tid < 64) hgg[tid] = h[(size_t)(8 * g + tid / 8) * in + 8 * g + tid % 8];
        if (tid < R * 8) bD[cur][tid / 8][0][tid % 8] = 0.f;
        if (tid < R * K && tid / K < nrows)
            bcode[cur][tid / K][0][tid % K] = codes_in[((size_t)(o0 + tid / K) * G + g) * K + tid % K];
        int nb = 1;
        __syncthreads();
#pragma unroll 1
        for (int k = 0; k < K; ++k) {
            const int nsel = (k == K - 1) ? 1 : beam;
            // per row and live beam: a = D_b - C_k[c0], const and w of the proposals
            for (int i = tid; i < R * nb; i += kEncThreads) {
                const int r = i / nb, b = i % nb;
                if (r >= nrows) continue;
                const uint32_t c0 = codes_in[((size_t)(o0 + r) * G + g) * K + k];
                float a[8], c0v[8];
                load_f8(cb[(size_t)k * 65536 + c0], c0v);
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = bD[cur][r][b][j] - c0v[j];
                float cst = 0.f;
#pragma unroll
                for (int ii = 0; ii < 8; ++ii) {
                    float t = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) t = fmaf(hgg[ii * 8 + j], a[j], t);
                    cst = fmaf(a[ii], t - 2.f * v[r][ii], cst);
                    bw[r][b][ii] = t - v[r][ii];
                }
                bconst[r][b] = cst;
            }
            uint64_t top[kEncMaxBeam];
#pragma unroll
            for (int i = 0; i < kEncMaxBeam; ++i) top[i] = ~0ull;
            uint64_t worst = ~0ull;  // top[nsel - 1]
            const float *qk = qtab + ((size_t)g * K + k) * 65536;
            const uint4 *cbk = cb + (size_t)k * 65536;
            // each thread moves kPer codewords and q values of a chunk; the
            // next chunk's are in flight (registers) while this one is scored
            constexpr int kPer = kE16Chunk / kEncThreads;
            uint4 nx[kPer];
            float nq[kPer];
#pragma unroll
            for (int p = 0; p < kPer; ++p) {
                nx[p] = cbk[tid + p * kEncThreads];
                nq[p] = qk[tid + p * kEncThreads];
            }
#pragma unroll 1
            for (int base = 0; base < 65536; base += kE16Chunk) {
                __syncthreads();  // the previous chunk is consumed (and bw, bconst written)
#pragma unroll
                for (int p = 0; p < kPer; ++p) {
                    float x[8];
                    load_f8(nx[p], x);
                    const int i = tid + p * kEncThreads;
#pragma unroll
                    for (int j = 0; j < 8; ++j) sx[i][j] = x[j];
                    sq[i] = nq[p];
                }
                if (base + kE16Chunk < 65536)
#pragma unroll
                    for (int p = 0; p < kPer; ++p) {
                        nx[p] = cbk[base + kE16Chunk + tid + p * kEncThreads];
                        nq[p] = qk[base + kE16Chunk + tid + p * kEncThreads];
                    }
                __syncthreads();
                if (my_r >= nrows) continue;
                auto offer = [&](uint64_t key) {
                    if (key < worst) {
                        // insert, dropping the largest; keep the list sorted
                        uint64_t x = key;
#pragma unroll
                        for (int i = 0; i < kEncMaxBeam; ++i)
                            if (i < nsel) {
                                const uint64_t lo = top[i] < x ? top[i] : x, hi = top[i] < x ? x : top[i];
                                top[i] = lo;
                                x = hi;
                            }
#pragma unroll
                        for (int i = 0; i < kEncMaxBeam; ++i)
                            if (i == nsel - 1) worst = top[i];
                    }
                };
                if (nb == 1) {
                    // one live beam (every slot of 1x16, the first of 2x16):
                    // its w and constant stay in registers
                    float wr[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) wr[j] = bw[my_r][0][j];
                    const float cst = bconst[my_r][0];
#pragma unroll 4
                    for (int c = my_s; c < kE16Chunk; c += S) {
                        float d = 0.f;
#pragma unroll
                        for (int j = 0; j < 8; ++j) d = fmaf(sx[c][j], wr[j], d);
                        offer(enc16_key(cst + sq[c] + 2.f * d, 0, base + c));
                    }
                } else {
#pragma unroll 1
                    for (int c = my_s; c < kE16Chunk; c += S) {
                        const float qc = sq[c];
#pragma unroll 1
                        for (int b = 0; b < nb; ++b) {
                            float d = 0.f;
#pragma unroll
                            for (int j = 0; j < 8; ++j) d = fmaf(sx[c][j], bw[my_r][b][j], d);
                            offer(enc16_key(bconst[my_r][b] + qc + 2.f * d, b, base + c));
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kEncMaxBeam; ++i) lists[my_r][my_s][i] = top[i];
            __syncthreads();
            // per row, the nsel smallest of its S sorted lists: warp w takes
            // rows w and w + 8, lane s < S holds list s's head
            for (int r = warp; r < R; r += kEncThreads / 32) {
                int head = 0;
                for (int t = 0; t < nsel; ++t) {
                    const uint64_t mine = (lane < S && head < kEncMaxBeam) ? lists[r][lane][head] : ~0ull;
                    const uint64_t m = warp_min_u64(mine);
                    if (lane < S && mine == m && m != ~0ull) ++head;
                    if (lane == 0) sel[r][t] = m;
                }
            }
            __syncthreads();
            const int nxt = cur ^ 1;
            for (int i = tid; i < R * nsel; i += kEncThreads) {
                const int r = i / nsel, t = i % nsel;
                if (r >= nrows) continue;
                const uint64_t key = sel[r][t];
                const int pb = (int)((key >> 16) & 0xff), c = (int)(key & 0xffff);
                const uint32_t c0 = codes_in[((size_t)(o0 + r) * G + g) * K + k];
                float cv[8], c0v[8];
                load_f8(cb[(size_t)k * 65536 + c], cv);
                load_f8(cb[(size_t)k * 65536 + c0], c0v);
#pragma unroll
                for (int j = 0; j < 8; ++j) bD[nxt][r][t][j] = bD[cur][r][pb][j] + cv[j] - c0v[j];
#pragma unroll
                for (int qq = 0; qq < K; ++qq) bcode[nxt][r][t][qq] = bcode[cur][r][pb][qq];
                bcode[nxt][r][t][k] = (uint16_t)c;
            }
            nb = nsel;
            cur = nxt;
            __syncthreads();
        }
        // commit each row's best beam
        for (int i = tid; i < nrows * 8; i += kEncThreads) {
            const int r = i / 8, j = i % 8;
            eg[(size_t)(o0 + r) * in + 8 * g + j] -= bD[cur][r][0][j];
        }
        for (int i = tid; i < nrows * K; i += kEncThreads)
            codes_out[((size_t)(o0 + i / K) * G + g) * K + i % K] = bcode[cur][i / K][0][i % K];
    }
}


}  // namespace aqk

namespace aqh {
using namespace aqk;

size_t encode_workspace_bytes(const Geom &g)
{
    if (g.B == 16)  // q table [G][K][65536] and the residual [out][in], fp32
        return kWsData + align16((size_t)g.G * g.K * 65536 * sizeof(float)) + (size_t)g.out * g.in * sizeof(float);
    return kWsData + align16((size_t)g.G * g.K * 256 * sizeof(float));
}

cudaError_t launch_encode(const Geom &g, const uint16_t *w, const float *h, const uint16_t *cb,
                          const void *codes_in, void *codes_out, int beam, void *ws, cudaStream_t s)
{
    float *q = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) + kWsData);
    const uint4 *c = reinterpret_cast<const uint4 *>(cb);
    const int smem = g.in * (int)sizeof(float);
    auto run = [&](auto kk) {
        constexpr int K = decltype(kk)::value;
        encode_q_kernel<K><<<g.G, 256, 0, s>>>(g.in, h, c, q);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(encode_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        encode_kernel<K><<<g.out, kEncThreads, smem, s>>>(g, w, h, c, q, reinterpret_cast<const uint8_t *>(codes_in),
                                                          reinterpret_cast<uint8_t *>(codes_out), beam);
        return cudaGetLastError();
    };
    if (g.B == 16) {
        float *eg = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) + kWsData +
                                              align16((size_t)g.G * g.K * 65536 * sizeof(float)));
        auto run16 = [&](auto kk) {
            constexpr int K = decltype(kk)::value;
            encode16_q_kernel<K><<<dim3(65536 / 256, g.G), 256, 0, s>>>(g.in, h, c, q);
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            constexpr int smem16 = encode16_smem_bytes();
            e = cudaFuncSetAttribute(encode16_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem16);
            if (e != cudaSuccess) return e;
            encode16_kernel<K><<<(g.out + kE16Rows - 1) / kE16Rows, kEncThreads, smem16, s>>>(
                g, w, h, c, q, reinterpret_cast<const uint16_t *>(codes_in), reinterpret_cast<uint16_t *>(codes_out),
                eg, beam);
            return cudaGetLastError();
        };
        if (g.K == 1) return run16(std::integral_constant<int, 1>{});
        if (g.K == 2) return run16(std::integral_constant<int, 2>{});
        return cudaErrorInvalidValue;
    }
    if (g.B != 8) return cudaErrorInvalidValue;
    if (g.K == 1) return run(std::integral_constant<int, 1>{});
    if (g.K == 2) return run(std::integral_constant<int, 2>{});
    if (g.K == 8) return run(std::integral_constant<int, 8>{});
    return cudaErrorInvalidValue;
}

}  // namespace aqh
