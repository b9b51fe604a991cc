// Shared device/host helpers of the sm_100a additive-quantised product library.
//
// Packed code layout (documented in include/aq.h): for each 8-row tile rt and
// each padded group g there is one chunk of 8 W bytes (W = K*B/8 bytes per
// word) holding the words of rows 8rt..8rt+7 for group g.  Chunk (rt, g)
// sits at chunk index rt*Gp + g, so 32 consecutive groups of one row tile
// are contiguous (512 bytes for the 2-bit schemes: one warp-wide 128-bit
// load).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/aq.h"

namespace aqk {

constexpr int kGroup = 8;        // weights per code group (in_group_size)
constexpr int kTileRows = 8;     // rows per packed chunk
constexpr int kGroupBlock = 32;  // groups per warp-wide load

// Streaming multiprocessors of a B200 (two dies of 74); launch plans size
// their grids in multiples of it.
constexpr int kNumSMs = 148;

struct Geom {
    int out, in, G;   // rows, columns, groups (in / 8)
    int K, B;         // codebooks, bits per code
    int rows8;        // rows padded to 8
    int gp;           // groups padded to 32
    int gblocks;      // gp / 32
    int rtiles;       // rows8 / 8
};

inline Geom make_geom(const aq_layer_desc &d)
{
    Geom g;
    g.out = d.out_features;
    g.in = d.in_features;
    g.G = d.in_features / kGroup;
    g.K = d.num_codebooks;
    g.B = d.nbits;
    g.rows8 = (g.out + 7) / 8 * 8;
    g.gp = (g.G + 31) / 32 * 32;
    g.gblocks = g.gp / 32;
    g.rtiles = g.rows8 / 8;
    return g;
}

inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }

// Workspace layout, the same for every entry point, so that one workspace
// serves any sequence of calls on a stream: status word at byte 0
// (AQ_ERR_TIMEOUT when a bounded wait gave up); split-K arrival counters in
// a fixed area of kWsMaxCounters words from byte 16, which only counters
// ever use and every call leaves at zero; the entry point's own data
// (split-K partial sums, tables) from kWsData on.  A plan splits a sum
// over CTAs only when its counters fit the area.
constexpr size_t kWsHeader = 16;
constexpr int kWsMaxCounters = 1024;
constexpr size_t kWsData = kWsHeader + sizeof(unsigned) * kWsMaxCounters;

// Atomic add with release and acquire semantics at GPU scope; returns the
// old value.
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned *p, unsigned v)
{
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void record_status(void *ws, uint32_t status)
{
    if (ws) atomicMax(reinterpret_cast<unsigned int *>(ws), status);
}

// binary16 pair helpers ------------------------------------------------------

__device__ __forceinline__ float2 h2f2(uint32_t v)
{
    __half2 h = *reinterpret_cast<__half2 *>(&v);
    return __half22float2(h);
}

__device__ __forceinline__ uint32_t f2h2(float a, float b)
{
    __half2 h = __floats2half2_rn(a, b);  // low half = a
    return *reinterpret_cast<uint32_t *>(&h);
}

// Sum of two binary16 8-vectors rounded once to binary16 (IEEE binary16
// addition, round to nearest even: the correctly rounded exact sum, signed
// zeros and overflow to infinity included).
__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b)
{
    __half2 r = __hadd2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint4 add_round_h8(uint4 a, uint4 b)
{
    return make_uint4(hadd2_u32(a.x, b.x), hadd2_u32(a.y, b.y), hadd2_u32(a.z, b.z),
                      hadd2_u32(a.w, b.w));
}

// s * w for eight binary16 w, rounded once (the fp32 product is exact).
__device__ __forceinline__ uint4 scale_round_h8(uint4 a, float s)
{
    uint4 r;
    float2 x;
    x = h2f2(a.x); r.x = f2h2(s * x.x, s * x.y);
    x = h2f2(a.y); r.y = f2h2(s * x.x, s * x.y);
    x = h2f2(a.z); r.z = f2h2(s * x.x, s * x.y);
    x = h2f2(a.w); r.w = f2h2(s * x.x, s * x.y);
    return r;
}

// Dot product of eight binary16 weights with eight binary16 activations,
// accumulated in fp32 onto acc.
__device__ __forceinline__ float dot8(uint4 w, uint4 x, float acc)
{
    float2 a, b;
    a = h2f2(w.x); b = h2f2(x.x); acc = fmaf(a.x, b.x, acc); acc = fmaf(a.y, b.y, acc);
    a = h2f2(w.y); b = h2f2(x.y); acc = fmaf(a.x, b.x, acc); acc = fmaf(a.y, b.y, acc);
    a = h2f2(w.z); b = h2f2(x.z); acc = fmaf(a.x, b.x, acc); acc = fmaf(a.y, b.y, acc);
    a = h2f2(w.w); b = h2f2(x.w); acc = fmaf(a.x, b.x, acc); acc = fmaf(a.y, b.y, acc);
    return acc;
}

// Read-only loads.  Not volatile: the compiler may hoist them, so that all
// independent gathers of a thread are in flight before the first use.
__device__ __forceinline__ uint4 ldg_nc_v4(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Release + acquire fence at GPU scope (orders this thread's, and by
// cumulativity its CTA's barrier-ordered, memory accesses against the next).
__device__ __forceinline__ void fence_acq_rel_gpu()
{
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Streaming load: read once, do not keep in L1.  Volatile, so a load
// written as a prefetch is issued where it is written rather than sunk by
// the compiler to its first use.
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Reduce acc[0..7] over the 32 lanes of a warp.  Afterwards lane l holds the
// total of row ((l>>4)&1)*4 + ((l>>3)&1)*2 + ((l>>2)&1).  9 shuffles.
__device__ __forceinline__ float warp_reduce8(float acc[8], int lane)
{
    const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4;
    float a4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float keep = h4 ? acc[i + 4] : acc[i];
        float send = h4 ? acc[i] : acc[i + 4];
        a4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float a2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float keep = h3 ? a4[i + 2] : a4[i];
        float send = h3 ? a4[i] : a4[i + 2];
        a2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float keep = h2 ? a2[1] : a2[0];
    float send = h2 ? a2[0] : a2[1];
    float v = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}

__device__ __forceinline__ int reduced_row_of_lane(int lane)
{
    return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
}

// ---------------------------------------------------------------------------
// mbarrier helpers with bounded waits (no wait in this library is unbounded).
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Non-blocking poll of a phase.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Poll a phase of an mbarrier at most `limit` times (each try_wait itself
// suspends for a hardware-defined interval).  Returns false on give-up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint32_t limit)
{
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

}  // namespace aqk

// Host-side launchers implemented in the kernel translation units.
namespace aqh {
cudaError_t launch_pack(const aqk::Geom &g, const void *codes, void *packed, cudaStream_t s);
cudaError_t launch_unpack(const aqk::Geom &g, const void *packed, void *codes, cudaStream_t s);
cudaError_t launch_dequant(const aqk::Geom &g, const void *packed, const uint16_t *cb,
                           const uint16_t *scales, uint16_t *w, cudaStream_t s);
size_t gemv_workspace_bytes(const aqk::Geom &g, int batch);
cudaError_t launch_gemv(const aqk::Geom &g, const void *packed, const uint16_t *cb,
                        const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                        void *ws, cudaStream_t s, bool pdl = true);
cudaError_t launch_gemv_noalloc(const aqk::Geom &g, const void *packed, const uint16_t *cb,
                                const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                                cudaStream_t s, bool *too_large);
size_t gemm_workspace_bytes(const aqk::Geom &g, int T);
cudaError_t launch_gemm(const aqk::Geom &g, const void *packed, const uint16_t *cb,
                        const uint16_t *scales, const uint16_t *x, int T, uint16_t *y,
                        void *ws, cudaStream_t s, bool pdl);
size_t param_grad_workspace_bytes(const aqk::Geom &g, int T);
cudaError_t launch_param_grad(const aqk::Geom &g, const void *packed, const uint16_t *cb, const uint16_t *scales,
                              const uint16_t *x, const uint16_t *gy, int T, float *grad_s, float *grad_cb,
                              void *ws, cudaStream_t s);
size_t encode_workspace_bytes(const aqk::Geom &g);
cudaError_t launch_encode(const aqk::Geom &g, const uint16_t *w, const float *h, const uint16_t *cb,
                          const void *codes_in, void *codes_out, int beam, void *ws, cudaStream_t s);
cudaError_t launch_selftest_wait(void *ws, int spin_limit, cudaStream_t s);
size_t gather_probe_sink_bytes(int mode);
cudaError_t launch_gather_probe(const uint16_t *codebook, const uint16_t *codes, size_t n, int mode, void *sink,
                                cudaStream_t s);
}  // namespace aqh
