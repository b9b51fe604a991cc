// C ABI of libaq_b200.so: argument validation and dispatch (see include/aq.h).
//
// Every entry point validates its arguments on the host before touching the
// GPU; on error nothing is launched.  No exception crosses the interface.
#include <stdint.h>

#include "scheme.cuh"

namespace {

using aqk::Geom;

constexpr int kVersion = 10000;  // 1.0.0
constexpr int32_t kMaxInFeatures = 65535 * 256;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Descriptor checks shared by all entry points.
aq_status check_desc(const aq_layer_desc *d)
{
    if (!d) return AQ_ERR_INVALID_ARG;
    if (d->out_features < 1 || d->in_features < 8 || d->in_features % 8) return AQ_ERR_INVALID_ARG;
    if (d->group_size != 8) return AQ_ERR_UNSUPPORTED;
    if (!aqk::scheme_supported(d->num_codebooks, d->nbits)) return AQ_ERR_UNSUPPORTED;
    // keep every byte offset and element count within 64-bit range and the
    // per-row chunk count within 32-bit kernel indices
    if ((int64_t)d->out_features * d->in_features > (int64_t)1 << 40) return AQ_ERR_INVALID_ARG;
    // grid.y of the split-K launches is at most 65535: the batch-1 table
    // path takes one split per block of 32 groups (in / 256 splits) and the
    // tensor path at most one per 4 stages of 8 groups (in / 256 again)
    if (d->in_features > kMaxInFeatures || d->out_features > (1 << 28)) return AQ_ERR_INVALID_ARG;
    return AQ_OK;
}

aq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA; }

}  // namespace

extern "C" {

const char *aq_status_string(aq_status status)
{
    switch (status) {
    case AQ_OK: return "success";
    case AQ_ERR_INVALID_ARG: return "invalid argument";
    case AQ_ERR_UNSUPPORTED: return "unsupported layer (scheme or group size)";
    case AQ_ERR_MISALIGNED: return "array pointer not 16-byte aligned";
    case AQ_ERR_WORKSPACE: return "workspace missing or too small";
    case AQ_ERR_CUDA: return "CUDA runtime error";
    case AQ_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    }
    return "unknown status";
}

int aq_version(void) { return kVersion; }

size_t aq_packed_codes_bytes(const aq_layer_desc *desc)
{
    if (check_desc(desc) != AQ_OK) return 0;
    const Geom g = aqk::make_geom(*desc);
    return (size_t)g.rows8 * g.gp * (g.K * g.B / 8);
}

size_t aq_gemv_workspace_bytes(const aq_layer_desc *desc, int batch)
{
    if (check_desc(desc) != AQ_OK || batch < 1 || batch > 16) return 0;
    return aqh::gemv_workspace_bytes(aqk::make_geom(*desc), batch);
}

size_t aq_gemm_workspace_bytes(const aq_layer_desc *desc, int T)
{
    if (check_desc(desc) != AQ_OK || T < 1) return 0;
    return aqh::gemm_workspace_bytes(aqk::make_geom(*desc), T);
}

aq_status aq_workspace_status(void *workspace, aq_stream_t stream)
{
    if (!workspace) return AQ_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return AQ_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return AQ_ERR_CUDA;
    if (word == 0) return AQ_OK;
    e = cudaMemsetAsync(workspace, 0, sizeof(word), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return AQ_ERR_CUDA;
    return word == AQ_ERR_TIMEOUT ? AQ_ERR_TIMEOUT : AQ_ERR_CUDA;
}

aq_status aq_selftest_bounded_wait(void *workspace, int spin_limit, aq_stream_t stream)
{
    if (!workspace || spin_limit < 1 || spin_limit > (1 << 20)) return AQ_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_selftest_wait(workspace, spin_limit, reinterpret_cast<cudaStream_t>(stream)));
}

aq_status aq_pack_codes(const aq_layer_desc *desc, const void *codes, void *packed, aq_stream_t stream)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (!codes || !packed) return AQ_ERR_INVALID_ARG;
    if (!aligned16(packed)) return AQ_ERR_MISALIGNED;
    if (desc->nbits == 16 && (reinterpret_cast<uintptr_t>(codes) & 1u)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_pack(aqk::make_geom(*desc), codes, packed,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

aq_status aq_unpack_codes(const aq_layer_desc *desc, const void *packed, void *codes, aq_stream_t stream)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (!codes || !packed) return AQ_ERR_INVALID_ARG;
    if (!aligned16(packed)) return AQ_ERR_MISALIGNED;
    if (desc->nbits == 16 && (reinterpret_cast<uintptr_t>(codes) & 1u)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_unpack(aqk::make_geom(*desc), packed, codes,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

aq_status aq_dequant(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                     const uint16_t *scales, uint16_t *w, aq_stream_t stream)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (!packed || !codebooks || !w) return AQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(codebooks) || !aligned16(w)) return AQ_ERR_MISALIGNED;
    if (scales && (reinterpret_cast<uintptr_t>(scales) & 1u)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_dequant(aqk::make_geom(*desc), packed, codebooks, scales, w,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

namespace {

aq_status gemv_entry(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                     const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                     void *workspace, size_t workspace_bytes, aq_stream_t stream, bool pdl)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (batch < 1 || batch > 16) return AQ_ERR_INVALID_ARG;
    if (!packed || !codebooks || !x || !y) return AQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(codebooks) || !aligned16(x) || !aligned16(y))
        return AQ_ERR_MISALIGNED;
    if (scales && (reinterpret_cast<uintptr_t>(scales) & 1u)) return AQ_ERR_MISALIGNED;
    const Geom g = aqk::make_geom(*desc);
    const size_t need = aqh::gemv_workspace_bytes(g, batch);
    if (!workspace || workspace_bytes < need) return AQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_gemv(g, packed, codebooks, scales, x, batch, y, workspace,
                                      reinterpret_cast<cudaStream_t>(stream), pdl));
}

}  // namespace

aq_status aq_gemv(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                  const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                  void *workspace, size_t workspace_bytes, aq_stream_t stream)
{
    return gemv_entry(desc, packed, codebooks, scales, x, batch, y, workspace, workspace_bytes, stream, true);
}

aq_status aq_gemv_ordered(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                          const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                          void *workspace, size_t workspace_bytes, aq_stream_t stream)
{
    return gemv_entry(desc, packed, codebooks, scales, x, batch, y, workspace, workspace_bytes, stream, false);
}

aq_status aq_gemv_noalloc(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                          const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                          aq_stream_t stream)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (batch < 1 || batch > 16) return AQ_ERR_INVALID_ARG;
    if (!packed || !codebooks || !x || !y) return AQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(codebooks) || !aligned16(x) || !aligned16(y))
        return AQ_ERR_MISALIGNED;
    if (scales && (reinterpret_cast<uintptr_t>(scales) & 1u)) return AQ_ERR_MISALIGNED;
    const Geom g = aqk::make_geom(*desc);
    bool too_large = false;
    const cudaError_t e = aqh::launch_gemv_noalloc(g, packed, codebooks, scales, x, batch, y,
                                                   reinterpret_cast<cudaStream_t>(stream), &too_large);
    if (too_large) return AQ_ERR_WORKSPACE;
    return from_cuda(e);
}

static aq_status gemm_entry(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                            const uint16_t *scales, const uint16_t *x, int T, uint16_t *y,
                            void *workspace, size_t workspace_bytes, aq_stream_t stream, bool pdl)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (T < 1 || T > (1 << 22)) return AQ_ERR_INVALID_ARG;  // grid.y = T/128 <= 32768
    if (!packed || !codebooks || !x || !y) return AQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(codebooks) || !aligned16(x) || !aligned16(y))
        return AQ_ERR_MISALIGNED;
    if (scales && (reinterpret_cast<uintptr_t>(scales) & 1u)) return AQ_ERR_MISALIGNED;
    const Geom g = aqk::make_geom(*desc);
    const size_t need = aqh::gemm_workspace_bytes(g, T);
    if (!workspace || workspace_bytes < need) return AQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_gemm(g, packed, codebooks, scales, x, T, y, workspace,
                                      reinterpret_cast<cudaStream_t>(stream), pdl));
}

aq_status aq_gemm(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                  const uint16_t *scales, const uint16_t *x, int T, uint16_t *y,
                  void *workspace, size_t workspace_bytes, aq_stream_t stream)
{
    return gemm_entry(desc, packed, codebooks, scales, x, T, y, workspace, workspace_bytes, stream, true);
}

aq_status aq_gemm_ordered(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                          const uint16_t *scales, const uint16_t *x, int T, uint16_t *y,
                          void *workspace, size_t workspace_bytes, aq_stream_t stream)
{
    return gemm_entry(desc, packed, codebooks, scales, x, T, y, workspace, workspace_bytes, stream, false);
}

size_t aq_encode_workspace_bytes(const aq_layer_desc *desc)
{
    if (check_desc(desc) != AQ_OK || desc->in_features > 16384) return 0;
    return aqh::encode_workspace_bytes(aqk::make_geom(*desc));
}

aq_status aq_encode(const aq_layer_desc *desc, const uint16_t *w, const float *h, const uint16_t *codebooks,
                    const void *codes_in, int beam, void *codes_out, void *workspace, size_t workspace_bytes,
                    aq_stream_t stream)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (desc->in_features > 16384 || beam < 1 || beam > 16) return AQ_ERR_INVALID_ARG;
    if (!w || !h || !codebooks || !codes_in || !codes_out || codes_in == codes_out) return AQ_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(h) || !aligned16(codebooks)) return AQ_ERR_MISALIGNED;
    const Geom g = aqk::make_geom(*desc);
    const size_t need = aqh::encode_workspace_bytes(g);
    if (!workspace || workspace_bytes < need) return AQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_encode(g, w, h, codebooks, codes_in, codes_out, beam, workspace,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

size_t aq_param_grad_workspace_bytes(const aq_layer_desc *desc, int T)
{
    if (check_desc(desc) != AQ_OK || T < 8 || T > (1 << 22) || T % 8) return 0;
    return aqh::param_grad_workspace_bytes(aqk::make_geom(*desc), T);
}

aq_status aq_param_grad(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                        const uint16_t *scales, const uint16_t *x, const uint16_t *gy, int T,
                        float *grad_scales, float *grad_codebooks, void *workspace,
                        size_t workspace_bytes, aq_stream_t stream)
{
    aq_status st = check_desc(desc);
    if (st != AQ_OK) return st;
    if (T < 8 || T > (1 << 22) || T % 8) return AQ_ERR_INVALID_ARG;
    if (!packed || !codebooks || !x || !gy) return AQ_ERR_INVALID_ARG;
    if (!aligned16(packed) || !aligned16(codebooks) || !aligned16(x) || !aligned16(gy) ||
        (grad_scales && !aligned16(grad_scales)) || (grad_codebooks && !aligned16(grad_codebooks)))
        return AQ_ERR_MISALIGNED;
    if (scales && (reinterpret_cast<uintptr_t>(scales) & 1u)) return AQ_ERR_MISALIGNED;
    const Geom g = aqk::make_geom(*desc);
    const size_t need = aqh::param_grad_workspace_bytes(g, T);
    if (!workspace || workspace_bytes < need) return AQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AQ_ERR_MISALIGNED;
    return from_cuda(aqh::launch_param_grad(g, packed, codebooks, scales, x, gy, T, grad_scales, grad_codebooks,
                                            workspace, reinterpret_cast<cudaStream_t>(stream)));
}

size_t aq_gather_probe_sink_bytes(int mode)
{
    if (mode < 0 || mode > 4) return 0;
    return aqh::gather_probe_sink_bytes(mode);
}

aq_status aq_gather_probe(const uint16_t *codebook, const uint16_t *codes, size_t n, int mode, void *sink,
                          aq_stream_t stream)
{
    if (mode < 0 || mode > 4) return AQ_ERR_INVALID_ARG;
    if ((mode != 3 && !codebook) || !codes || !sink || n == 0 || n % 8 || n > ((size_t)1 << 36))
        return AQ_ERR_INVALID_ARG;
    if ((codebook && !aligned16(codebook)) || !aligned16(codes) || !aligned16(sink)) return AQ_ERR_MISALIGNED;
    return from_cuda(
        aqh::launch_gather_probe(codebook, codes, n, mode, sink, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
