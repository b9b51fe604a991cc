// Codeword-read ceiling of the 1x16 decode-time product (a measurement aid,
// not part of the product path).
//
// The 1x16 GEMV is bound by random 16-byte reads from the 1 MiB codebook
// (65536 codewords of 8 binary16 weights), one read per code.  These kernels
// issue the same reads and nothing else, so their time is the ceiling the
// GEMV is measured against:
//  * mode 0 (L2, the route of the GEMV's decoders): two CTAs of 128 threads
//    per SM; per stage each thread takes one 16-byte chunk of 8 codes and
//    copies their codewords with cp.async into its slots of a 5-stage
//    shared-memory ring, three stages in flight, then folds the landed
//    stage into a checksum;
//  * mode 1 (distributed shared memory): clusters of 8 CTAs, each holding
//    one eighth of the codebook (128 KiB) in shared memory, loaded once per
//    launch; every codeword is read from its owner's shared memory with
//    ld.shared::cluster, a chunk's 8 reads in flight;
//  * mode 2 (registers through L1, the route of the batch-1 CUDA-core
//    GEMV): three CTAs of 256 threads per SM, a chunk's 8 codewords read
//    with ld.global.nc into registers, no shared memory (L1 keeps what it
//    can of the codebook).
//  * mode 4 (codebook slices, work moved to the slice): clusters of 8 CTAs
//    of 512 threads, each holding one eighth of the codebook (128 KiB) in
//    its own shared memory; every CTA of a cluster reads the cluster's code
//    chunks (from L2: each chunk is read by the cluster's 8 CTAs) and
//    handles only the codes whose top 3 bits name its slice, with local
//    shared-memory reads.  The route a 1x16 product would take if it kept
//    the codebook on chip and reduced the 8 CTAs' partial sums through
//    distributed shared memory once per row tile.
//  * mode 3 (read-only HBM stream, the cross-check of the copy bandwidth
//    the HBM roofline uses): the `codes` array itself is read once, 16
//    bytes per load, eight loads in flight per thread, four CTAs of 256
//    threads per SM, L1 bypassed; no codebook read.  Over an array much
//    larger than L2 its time is the read bandwidth of HBM.
// Each thread XORs every 32-bit word it reads into a 16-byte checksum
// written to `sink` (so the reads cannot be elided, and a test can compare
// the XOR of all checksums with the XOR of the codewords the codes select).
#include "aq_common.cuh"
#include "tc_common.cuh"

namespace aqk {

constexpr int kProbeThreads = 128;
constexpr int kProbeRing = 5;   // stages of the shared-memory ring (mode 0)
constexpr int kProbeLag = 3;    // stages in flight (mode 0)
constexpr int kClusterCtas = 8;  // mode 1
constexpr int kSliceWords = 65536 / kClusterCtas;

__device__ __forceinline__ void xor_into(uint4 &a, uint4 v)
{
    a.x ^= v.x;
    a.y ^= v.y;
    a.z ^= v.z;
    a.w ^= v.w;
}

__device__ __forceinline__ uint32_t code_of(uint4 w, int j)
{
    const uint32_t u = (j < 2) ? w.x : (j < 4) ? w.y : (j < 6) ? w.z : w.w;
    return (u >> (16 * (j & 1))) & 0xffffu;
}

// Chunk q of the n / 8 chunks for thread (CTA c, thread t) at step k:
// (k * gridDim + c) * blockDim + t, so a warp reads 512 consecutive bytes.
__global__ void __launch_bounds__(kProbeThreads)
probe_l2_kernel(const uint4 *__restrict__ cb, const uint4 *__restrict__ chunks, long nchunks, uint4 *sink)
{
    extern __shared__ uint4 ring[];  // [kProbeRing][8][kProbeThreads]
    const int t = threadIdx.x;
    const long stride = (long)gridDim.x * kProbeThreads;
    const long first = (long)blockIdx.x * kProbeThreads + t;
    const int steps = first < nchunks ? (int)((nchunks - 1 - first) / stride + 1) : 0;
    grid_launch_dependents();
    uint4 acc = make_uint4(0u, 0u, 0u, 0u);
    auto slot = [&](int i, int j) { return smem_u32(ring + (((i % kProbeRing) * 8 + j) * kProbeThreads + t)); };
    for (int i = 0; i < steps + kProbeLag; ++i) {
        if (i < steps) {
            const uint4 w = ldg_stream_v4(chunks + first + (long)i * stride);
#pragma unroll
            for (int j = 0; j < 8; ++j) cp_async16(slot(i, j), cb + code_of(w, j), 16u);
        }
        cp_async_commit();
        const int d = i - kProbeLag;  // its copies have landed once kProbeLag newer groups are pending
        if (d >= 0) {
            cp_async_wait<kProbeLag>();
            if (d < steps) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 v;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(slot(d, j)));
                    xor_into(acc, v);
                }
            }
        }
    }
    cp_async_wait<0>();
    grid_dependency_wait();  // the previous launch on the stream may still write the sink
    sink[first] = acc;
}

constexpr int kProbeLdgThreads = 256;
constexpr int kProbeLdgPerSM = 3;

__global__ void __launch_bounds__(kProbeLdgThreads, kProbeLdgPerSM)
probe_ldg_kernel(const uint4 *__restrict__ cb, const uint4 *__restrict__ chunks, long nchunks, uint4 *sink)
{
    const long stride = (long)gridDim.x * kProbeLdgThreads;
    const long first = (long)blockIdx.x * kProbeLdgThreads + threadIdx.x;
    grid_launch_dependents();
    uint4 acc = make_uint4(0u, 0u, 0u, 0u);
    for (long q = first; q < nchunks; q += stride) {
        const uint4 w = ldg_stream_v4(chunks + q);
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = ldg_nc_v4(cb + code_of(w, j));
#pragma unroll
        for (int j = 0; j < 8; ++j) xor_into(acc, v[j]);
    }
    grid_dependency_wait();  // the previous launch on the stream may still write the sink
    sink[first] = acc;
}

constexpr int kProbeStreamThreads = 256;
constexpr int kProbeStreamPerSM = 4;
constexpr int kProbeStreamUnroll = 8;

// Thread (CTA c, thread t) reads chunks q = base + u * stride for u < 8,
// base = (k * gridDim + c) * 8 * blockDim + t at step k: every load
// instruction of a warp reads 512 consecutive bytes.
__global__ void __launch_bounds__(kProbeStreamThreads, kProbeStreamPerSM)
probe_stream_kernel(const uint4 *__restrict__ chunks, long nchunks, uint4 *sink)
{
    const long per_step = (long)gridDim.x * kProbeStreamThreads * kProbeStreamUnroll;
    const long first = (long)blockIdx.x * kProbeStreamThreads + threadIdx.x;
    const long cta0 = (long)blockIdx.x * kProbeStreamThreads * kProbeStreamUnroll + threadIdx.x;
    grid_launch_dependents();
    uint4 acc = make_uint4(0u, 0u, 0u, 0u);
    long q0 = cta0;
    for (; q0 + (long)(kProbeStreamUnroll - 1) * kProbeStreamThreads < nchunks; q0 += per_step) {
        uint4 v[kProbeStreamUnroll];
#pragma unroll
        for (int u = 0; u < kProbeStreamUnroll; ++u) v[u] = ldg_stream_v4(chunks + q0 + (long)u * kProbeStreamThreads);
#pragma unroll
        for (int u = 0; u < kProbeStreamUnroll; ++u) xor_into(acc, v[u]);
    }
    for (int u = 0; u < kProbeStreamUnroll; ++u) {  // the ragged last step
        const long q = q0 + (long)u * kProbeStreamThreads;
        if (q < nchunks) xor_into(acc, ldg_stream_v4(chunks + q));
    }
    grid_dependency_wait();  // the previous launch on the stream may still write the sink
    sink[first] = acc;
}

constexpr int kProbeSliceThreads = 512;

__global__ void __launch_bounds__(kProbeSliceThreads, 1)
probe_slice_kernel(const uint4 *__restrict__ cb, const uint4 *__restrict__ chunks, long nchunks, uint4 *sink)
{
    extern __shared__ uint4 slice_words[];  // codewords [rank * kSliceWords, (rank + 1) * kSliceWords)
    const int t = threadIdx.x;
    const uint32_t rank = cluster_ctarank();
    const long cluster = blockIdx.x / kClusterCtas, nclusters = gridDim.x / kClusterCtas;
    for (int i = t; i < kSliceWords; i += kProbeSliceThreads)
        cp_async16(smem_u32(slice_words + i), cb + (size_t)rank * kSliceWords + i, 16u);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    grid_launch_dependents();
    // chunk q of the cluster's share, the same sequence in its 8 CTAs
    const long stride = nclusters * kProbeSliceThreads;
    uint4 acc = make_uint4(0u, 0u, 0u, 0u);
    for (long q = cluster * kProbeSliceThreads + t; q < nchunks; q += stride) {
        const uint4 w = ldg_stream_v4(chunks + q);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t c = code_of(w, j);
            if ((c >> 13) == rank) xor_into(acc, slice_words[c & (kSliceWords - 1)]);
        }
    }
    grid_dependency_wait();  // the previous launch on the stream may still write the sink
    sink[(long)blockIdx.x * kProbeSliceThreads + t] = acc;
}

__global__ void __launch_bounds__(kProbeThreads)
probe_dsmem_kernel(const uint4 *__restrict__ cb, const uint4 *__restrict__ chunks, long nchunks, uint4 *sink)
{
    extern __shared__ uint4 slice[];  // codewords [rank * kSliceWords, (rank + 1) * kSliceWords)
    const int t = threadIdx.x;
    const uint32_t rank = cluster_ctarank();
    for (int i = t; i < kSliceWords; i += kProbeThreads)
        cp_async16(smem_u32(slice + i), cb + (size_t)rank * kSliceWords + i, 16u);
    cp_async_commit();
    cp_async_wait<0>();
    cluster_sync_all();  // every slice of the cluster is loaded
    grid_launch_dependents();
    const uint32_t base = smem_u32(slice);
    const long stride = (long)gridDim.x * kProbeThreads;
    const long first = (long)blockIdx.x * kProbeThreads + t;
    uint4 acc = make_uint4(0u, 0u, 0u, 0u);
    for (long q = first; q < nchunks; q += stride) {
        const uint4 w = ldg_stream_v4(chunks + q);
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t c = code_of(w, j);
            v[j] = ld_peer_shared(base + (c % kSliceWords) * 16u, c / kSliceWords);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) xor_into(acc, v[j]);
    }
    cluster_sync_all();  // no CTA leaves while another still reads its slice
    grid_dependency_wait();
    sink[first] = acc;
}

}  // namespace aqk

namespace aqh {
using namespace aqk;

namespace {

int probe_l2_ctas() { return 2 * kNumSMs; }

// CTAs of whole 8-CTA clusters that run at once (mode 1: 128 threads,
// mode 4: 512), at most one per SM
cudaError_t probe_cluster_ctas(int mode, int *ctas)
{
    const int smem = kSliceWords * 16;
    const void *kern = mode == 4 ? (const void *)probe_slice_kernel : (const void *)probe_dsmem_kernel;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterCtas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(kClusterCtas);
    cfg.blockDim = dim3(mode == 4 ? kProbeSliceThreads : kProbeThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    *ctas = std::min(std::max(1, clusters) * kClusterCtas, kNumSMs / kClusterCtas * kClusterCtas);
    return cudaSuccess;
}

}  // namespace

size_t gather_probe_sink_bytes(int mode)
{
    // mode 1 runs at most one CTA per SM (128 KiB of shared memory each)
    if (mode == 2) return (size_t)kProbeLdgPerSM * kNumSMs * kProbeLdgThreads * sizeof(uint4);
    if (mode == 3) return (size_t)kProbeStreamPerSM * kNumSMs * kProbeStreamThreads * sizeof(uint4);
    if (mode == 4) return (size_t)kNumSMs * kProbeSliceThreads * sizeof(uint4);
    const int ctas = mode == 0 ? probe_l2_ctas() : kNumSMs;
    return (size_t)ctas * kProbeThreads * sizeof(uint4);
}

cudaError_t launch_gather_probe(const uint16_t *codebook, const uint16_t *codes, size_t n, int mode, void *sink,
                                cudaStream_t s)
{
    const uint4 *cb = reinterpret_cast<const uint4 *>(codebook);
    const uint4 *chunks = reinterpret_cast<const uint4 *>(codes);
    const long nchunks = (long)(n / 8);
    uint4 *out = reinterpret_cast<uint4 *>(sink);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kProbeThreads);
    cfg.stream = s;
    cfg.attrs = attr;
    cudaError_t e;
    if (mode == 3) {
        cfg.gridDim = dim3(kProbeStreamPerSM * kNumSMs);
        cfg.blockDim = dim3(kProbeStreamThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, probe_stream_kernel, chunks, nchunks, out);
    } else if (mode == 2) {
        cfg.gridDim = dim3(kProbeLdgPerSM * kNumSMs);
        cfg.blockDim = dim3(kProbeLdgThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, probe_ldg_kernel, cb, chunks, nchunks, out);
    } else if (mode == 0) {
        const int smem = kProbeRing * 8 * kProbeThreads * (int)sizeof(uint4);
        e = cudaFuncSetAttribute(probe_l2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(probe_l2_ctas());
        cfg.dynamicSmemBytes = smem;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, probe_l2_kernel, cb, chunks, nchunks, out);
    } else {
        // modes 1 and 4: whole 8-CTA clusters, at most one CTA per SM (the
        // sink holds one CTA per SM)
        int ctas = 0;
        e = probe_cluster_ctas(mode, &ctas);
        if (e != cudaSuccess) return e;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = kClusterCtas;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.gridDim = dim3(ctas);
        cfg.dynamicSmemBytes = kSliceWords * 16;
        cfg.numAttrs = 2;
        if (mode == 4) {
            cfg.blockDim = dim3(kProbeSliceThreads);
            e = cudaLaunchKernelEx(&cfg, probe_slice_kernel, cb, chunks, nchunks, out);
        } else {
            e = cudaLaunchKernelEx(&cfg, probe_dsmem_kernel, cb, chunks, nchunks, out);
        }
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace aqh
