/*
 * aq.h -- C ABI of the B200 (sm_100a) additive-quantised matrix product
 * library (libaq_b200.so).
 *
 * What it computes.  The additive quantisation of "Extreme Compression of
 * Large Language Models via Additive Quantization" (Egiazarian et al., ICML
 * 2024) stores each group of 8 consecutive input weights of one output row
 * as K codes; the group is rebuilt as the sum of one 8-vector from each of K
 * codebooks (AQLM wiki entry, brain.gartu.xyz, section "Niveau
 * intermédiaire": w ~ C_1[i_1] + ... + C_K[i_K]; devtrends.ru summary
 * "AQLM — Сжимаем языковые модели без потерь", section "Как это работает
 * технически?": groups of 8, in_group_size).  With K codebooks of 2^B
 * entries the bit rate is K*B/8 bits per weight ("Niveau intermédiaire",
 * bit-rate formula).  The library multiplies the decoded matrix by
 * activations, the operation the paper's abstract (arXiv 2401.06118) names
 * for token generation, with one scale per output row:
 *
 *     W[o][8g+j] = RN16( sum_k C_k[codes[o][g][k]][j] )          (decode)
 *     y[o][b]    = RN16( s[o] * sum_i W[o][i] * x[i][b] )        (product)
 *
 * Supported schemes (K x B): "1x16" and "2x8" (2 bits per weight) and
 * "8x8" (8 bits per weight), named in devtrends.ru, section "Схемы
 * квантования"; "2x16" (4 bits per weight), the AQLM wiki entry's example in
 * "Niveau intermédiaire"; "1x8" (1 bit per weight), devtrends.ru's notes on
 * 1-bit models.  Codes are uint8 for B = 8 and uint16 for B = 16.
 *
 * Conventions shared by every entry point:
 *  - binary16 values are passed as uint16_t bit patterns (IEEE 754 half);
 *  - every array pointer is a DEVICE pointer on the current CUDA device,
 *    owned by the caller; the library allocates no memory and keeps no
 *    state between calls (thread-safe; calls on one stream are ordered),
 *    except aq_gemv_noalloc, which uses one fixed device array of the
 *    library (described at that function);
 *  - work is enqueued on `stream` (NULL = legacy default stream) and the
 *    call returns after the launch; the caller synchronises;
 *  - the GEMV kernels use programmatic dependent launch: a GEMV may start
 *    reading its weights (packed codes, codebooks) while the GEMV launched
 *    just before it on the stream is still running; it reads x and writes
 *    y and the workspace only after that launch has completed.  GEMVs write
 *    no weights, and other kernels (this library's or the caller's) let the
 *    next launch start only when they complete, so stream order holds for
 *    every value a caller can observe;
 *  - all arguments are validated on the host before anything is launched;
 *    on any error status nothing is launched and no output byte is written;
 *  - array pointers must be 16-byte aligned (AQ_ERR_MISALIGNED otherwise);
 *  - no C++ exception crosses this interface.
 *
 * Packed code layout (produced by aq_pack_codes, consumed by every kernel).
 * Each group (o, g) owns one word of W = K*B/8 bytes holding its K codes,
 * code k in bits [k*B, (k+1)*B) (1x16: the code; 2x8: c0 | c1 << 8; 1x8:
 * one byte; 2x16: c0 | c1 << 16; 8x8: eight bytes, c0 first).  Rows are
 * padded to a multiple of 8 and groups to a multiple of 32 (Gp = padded
 * group count); padding words are zero.  Word (o, g) is stored
 * little-endian at byte
 *
 *     ((o / 8) * (Gp / 32) + g / 32) * 256 W  +  (g % 32) * 8 W  +  (o % 8) * W
 *
 * i.e. 256 W-byte tiles of 8 rows x 32 groups, tile-rows in row order;
 * inside a tile the 8 W-byte chunk c holds group 32*(g/32)+c for the
 * tile's 8 rows (for the 2-bit schemes a 16-byte chunk, so one warp-wide
 * 128-bit load fetches a whole tile).
 */
#ifndef AQ_B200_H
#define AQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a pointer to the runtime's opaque stream). */
struct CUstream_st;
typedef struct CUstream_st *aq_stream_t;

typedef enum {
    AQ_OK = 0,
    AQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, in % 8 != 0, ...     */
    AQ_ERR_UNSUPPORTED = 2, /* (K, B) or group size the library cannot run */
    AQ_ERR_MISALIGNED = 3,  /* an array pointer not 16-byte aligned         */
    AQ_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required   */
    AQ_ERR_CUDA = 5,        /* the CUDA runtime reported an error           */
    AQ_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up           */
} aq_status;

/* One quantised linear layer: y[out] = diag(s) W[out][in] x[in]. */
typedef struct {
    int32_t out_features;  /* rows of W, 1 .. 2^28                         */
    int32_t in_features;   /* columns of W, 8 .. 65535*256, multiple of 8  */
    int32_t group_size;    /* weights per code group; must be 8            */
    int32_t num_codebooks; /* K: 1x16, 2x8, 1x8, 2x16 or 8x8 with nbits    */
    int32_t nbits;         /* B: bits per code, codebook has 2^B entries   */
} aq_layer_desc;

/* Static, NUL-terminated description of a status; never NULL. */
const char *aq_status_string(aq_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int aq_version(void);

/*
 * Bytes of the packed code buffer for `desc` (layout above): padded rows x
 * padded groups x 2.  Returns 0 for an invalid or unsupported descriptor.
 * Host-only; needs no GPU.
 */
size_t aq_packed_codes_bytes(const aq_layer_desc *desc);

/*
 * Workspace.  aq_gemv, aq_gemm, aq_param_grad and aq_encode take a
 * caller-owned device workspace.  Its first 16 bytes hold a status word that
 * a kernel sets when a bounded wait gives up (read it with
 * aq_workspace_status); then come split-K arrival counters in a fixed area
 * of 4 KiB, then the call's own data (split-K partial sums, tables).  A
 * workspace must be zero-filled once before its first use; every completed
 * call leaves it ready for the next (counters back at zero), whatever the
 * layer or entry point, so one workspace as large as the largest size any
 * of the calls needs serves a whole sequence of calls on one stream (all
 * the linears of a model, for instance).  Calls that may overlap in time
 * (different streams) must not share a workspace.
 *
 * The sizes below are host-only (no GPU needed) and depend on the
 * descriptor and batch / token count alone.  They return 0 for invalid
 * arguments, never less than 16 otherwise.
 */
size_t aq_gemv_workspace_bytes(const aq_layer_desc *desc, int batch);
size_t aq_gemm_workspace_bytes(const aq_layer_desc *desc, int T);

/*
 * Read and clear the status word of `workspace` after all work queued on
 * `stream` has finished (this call synchronises `stream`).  Returns AQ_OK,
 * AQ_ERR_TIMEOUT if a kernel's bounded wait gave up since the last read, or
 * AQ_ERR_CUDA.
 */
aq_status aq_workspace_status(void *workspace, aq_stream_t stream);

/*
 * Test aid for failure detection: launches one CTA that waits on a barrier
 * nothing will ever complete, gives up after `spin_limit` polls, records
 * AQ_ERR_TIMEOUT in the workspace status word and returns.  The context
 * stays usable.  spin_limit in 1..1<<20.
 */
aq_status aq_selftest_bounded_wait(void *workspace, int spin_limit, aq_stream_t stream);

/*
 * Interleave codes into the packed layout (offline, once per layer).
 *   codes  [out][in/8][K]: uint8 for B = 8, uint16 for B = 16 (row-major).
 *   packed aq_packed_codes_bytes(desc) bytes; every byte is written,
 *          padding included.
 * `codes` needs only the alignment of its element type; `packed` 16 bytes.
 */
aq_status aq_pack_codes(const aq_layer_desc *desc, const void *codes, void *packed,
                        aq_stream_t stream);

/* Inverse of aq_pack_codes (a test aid): packed -> codes[out][in/8][K]. */
aq_status aq_unpack_codes(const aq_layer_desc *desc, const void *packed, void *codes,
                          aq_stream_t stream);

/*
 * Dequantise: w[o][i] = RN16(sum_k C_k[codes[o][g][k]][i - 8g]) with
 * g = i / 8, or, when `scales` is not NULL, RN16(s[o] * that value).  The sum
 * is rounded once (round to nearest, ties to even) and matches the exact sum
 * bit for bit.
 *   packed    aq_packed_codes_bytes(desc) bytes (from aq_pack_codes)
 *   codebooks [K][2^B][8] binary16
 *   scales    [out] binary16 or NULL
 *   w         [out][in] binary16, row-major (written in full)
 */
aq_status aq_dequant(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                     const uint16_t *scales, uint16_t *w, aq_stream_t stream);

/*
 * Decode-time product for batch 1..16:
 *   y[o][b] = RN16(s[o] * sum_i W[o][i] x[i][b]), fp32 accumulation.
 *   packed    from aq_pack_codes
 *   codebooks [K][2^B][8] binary16
 *   scales    [out] binary16, or NULL for s = 1
 *   x         [in][batch] binary16, row-major
 *   y         [out][batch] binary16, row-major (written in full)
 *   workspace >= aq_gemv_workspace_bytes(desc, batch) bytes (see above)
 * Results are deterministic: the same inputs give the same bits.
 * AQ_ERR_INVALID_ARG for batch outside 1..16.
 * Early weight reads: this kernel is launched with programmatic dependent
 * launch and may read `packed` and `codebooks` before the kernel launched
 * just before it on `stream` has finished (x, scales, y and the workspace
 * only after).  That is safe whenever the previous kernel does not write
 * this layer's packed codes or codebooks, or does not let its dependents
 * start early (griddepcontrol.launch_dependents / cudaTriggerProgrammatic-
 * LaunchCompletion) -- every kernel of this library and every kernel that
 * does not use programmatic launch qualifies.  A caller whose own kernel
 * triggers its dependents early and then rewrites these weights (a
 * fine-tuning step, for instance) must write them before the trigger, or
 * call aq_gemv_ordered instead.
 */
aq_status aq_gemv(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                  const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                  void *workspace, size_t workspace_bytes, aq_stream_t stream);

/*
 * aq_gemv with an ordinary launch: the kernel starts only after all work
 * queued before it on `stream` has completed, so it reads no weight early.
 * Same arguments, plan and results (bit for bit) as aq_gemv; it gives up
 * the overlap of a launch with the end of the previous one.
 */
aq_status aq_gemv_ordered(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                          const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                          void *workspace, size_t workspace_bytes, aq_stream_t stream);

/*
 * aq_gemv without a workspace argument, for callers that cannot allocate
 * device memory: code that runs where the host framework owns every device
 * allocation, real-time loops that forbid allocation after start-up, or
 * plugins handed only input and output buffers.  The paper has no
 * counterpart; this is an interface convenience.
 *
 * Same arguments and results as aq_gemv, minus the workspace (including
 * aq_gemv's rule on early weight reads).  Where
 * aq_gemv's split-K partial sums would not fit the scratch, this call splits
 * the sum more coarsely (on the tensor-core path, down to one CTA per 128
 * rows, which needs no partial sums; 8-bit codebooks at batch 1 then leave
 * the table path for the tensor-core path), so its y agrees with aq_gemv's
 * within rounding rather than bit for bit; it is deterministic run to run.
 * The split-K scratch is a fixed device array inside the library of
 * AQ_GEMV_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the
 * library holds until the process exits.  The call allocates nothing (no
 * cudaMalloc/cudaFree, no allocating library routine); it clears the part
 * of the array that must start at zero with cudaMemsetAsync on `stream`.
 *  - The first call in each CUDA context of a device (the device's primary
 *    context, or a context the caller made current) looks up the array's
 *    device address (cudaGetSymbolAddress, with that device current) and
 *    keeps it with the context's id; make that first call before any stream
 *    capture on that device.  After cudaDeviceReset or under another
 *    context the next call looks the address up again.
 *  - Every call shares the one array and it keeps the last call's contents:
 *    calls whose kernels may overlap on the GPU (different streams) race and
 *    give wrong results.  Serialise them, or use aq_gemv with a workspace
 *    per stream.
 *  - AQ_ERR_WORKSPACE if the layer would need more scratch than the array
 *    holds even at the coarsest split; nothing is launched then.  The
 *    coarsest split (one CTA per 128 rows) needs no partial sums and no
 *    counters, so no layer the descriptor limits allow reaches this today;
 *    the status stays as the contract for plans that might.
 *  - A bounded wait that gives up inside the kernel cannot be reported (the
 *    status word is internal): use aq_gemv when that report is needed.
 */
#define AQ_GEMV_NOALLOC_SCRATCH_BYTES (4u << 20)
aq_status aq_gemv_noalloc(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                          const uint16_t *scales, const uint16_t *x, int batch, uint16_t *y,
                          aq_stream_t stream);

/*
 * Prefill product for 1 <= T <= 2^22 tokens on the tensor cores (tcgen05.mma with
 * binary16 operands and fp32 accumulation in tensor memory):
 *   y[o][t] = RN16(s[o] * sum_i W[o][i] x[i][t]).
 *   x [in][T] binary16 row-major; y [out][T] binary16 row-major; other
 *   arguments as for aq_gemv; workspace >= aq_gemm_workspace_bytes(desc, T).
 * Every wait inside the kernel is bounded: if one gives up, the kernel
 * records AQ_ERR_TIMEOUT in the workspace status word (see
 * aq_workspace_status), frees its tensor memory and returns; the output is
 * then incomplete but the context stays usable.
 * Early weight reads: for T a multiple of 8 the kernel is launched with
 * programmatic dependent launch, as aq_gemv is, and may read `packed` and
 * `codebooks` before the kernel launched just before it on `stream` has
 * finished (x, scales, y and the workspace only after); aq_gemv's rule on
 * early weight reads applies, and aq_gemm_ordered is the ordinary launch.
 */
aq_status aq_gemm(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                  const uint16_t *scales, const uint16_t *x, int T, uint16_t *y,
                  void *workspace, size_t workspace_bytes, aq_stream_t stream);

/*
 * aq_gemm with an ordinary launch: the kernel starts only after all work
 * queued before it on `stream` has completed, so it reads no weight early.
 * Same arguments, plan and results (bit for bit) as aq_gemm.
 */
aq_status aq_gemm_ordered(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                          const uint16_t *scales, const uint16_t *x, int T, uint16_t *y,
                          void *workspace, size_t workspace_bytes, aq_stream_t stream);

/*
 * Parameter gradient of a quantised layer: for the loss L = sum(gy * y) with
 * y = diag(s) W x (the product of aq_gemm), the gradients with respect to
 * the row scales and the codebook entries, which the step that fine-tunes
 * the codebooks after the codes are fixed needs (AQLM wiki entry, "Niveau
 * tech avancé": codebooks learned jointly with the codes by minimising the
 * layer's output error).  The decode's binary16 rounding is taken as the
 * identity, so with M[o][i] = sum_b gy[o][b] x[i][b]:
 *
 *     grad_scales[o]          = sum_i W[o][i] M[o][i]
 *     grad_codebooks[k][c][j] = sum of s[o] M[o][8g+j] over the groups (o, g)
 *                               whose code k is c          (s = 1 if NULL)
 *
 *   x              [in][T]  binary16 (the layer input),
 *   gy             [out][T] binary16 (dL/dy),
 *   T              tokens, 8..1<<22 and a multiple of 8 (the rows of x and
 *                  gy are read by TMA, whose row pitch must be a multiple of
 *                  16 bytes; pad with zero tokens otherwise),
 *   grad_scales    [out] fp32, overwritten; NULL to skip,
 *   grad_codebooks [K][2^B][8] fp32, overwritten; NULL to skip,
 *   workspace      >= aq_param_grad_workspace_bytes(desc, T) bytes (status
 *                  word; AQ_ERR_TIMEOUT there if a bounded wait gave up).
 * The sums are accumulated with fp32 atomic adds: their order, and so the
 * last bits of the result, may change from run to run.
 */
/*
 * Encoder: beam search of the codes for fixed codebooks under the
 * quantisation objective of the AQLM wiki entry ("Niveau tech avancé"),
 * || W - sum_k C_k[i_k] ||^2_H with H = 2 X^T X.  The objective is a sum
 * over output rows of e^T H e (e = w - reconstruction), so rows are
 * independent.  Per row, groups in order with the others fixed, a beam of
 * width `beam` runs over the group's K codes, codebook by codebook: every
 * beam proposes each code for the slot, the `beam` proposals with the
 * smallest objective survive (ties: parent beam, then code), and the best
 * beam is kept before the next group.  The reconstruction is the exact
 * codeword sum; arithmetic is fp32.
 *   w          [out][in] binary16 (the weights to approximate),
 *   h          [in][in] fp32, symmetric (e.g. 2 X^T X of calibration
 *              activations),
 *   codes_in   [out][in/8][K] uint8 (B = 8) or uint16 (B = 16): the
 *              starting codes,
 *   codes_out  the same shape and type, written (may not alias codes_in),
 *   beam       1..16,
 *   workspace  >= aq_encode_workspace_bytes(desc) bytes (a per-layer table
 *              of C_k[c]^T H_gg C_k[c]; for B = 16 also the rows' residual
 *              w - reconstruction, [out][in] fp32).
 * Every scheme (1x8, 2x8, 8x8, 1x16, 2x16); in <= 16384.  For B = 16 the
 * search scores all 65536 codes of each slot (one CTA per 16 rows, the
 * codebook streamed through shared memory): with one codebook the beam
 * keeps nothing past the group's best proposal, so any beam gives the
 * codes of beam 1; with two, the first slot keeps `beam` proposals.
 */
size_t aq_encode_workspace_bytes(const aq_layer_desc *desc);
aq_status aq_encode(const aq_layer_desc *desc, const uint16_t *w, const float *h, const uint16_t *codebooks,
                    const void *codes_in, int beam, void *codes_out, void *workspace, size_t workspace_bytes,
                    aq_stream_t stream);

size_t aq_param_grad_workspace_bytes(const aq_layer_desc *desc, int T);
aq_status aq_param_grad(const aq_layer_desc *desc, const void *packed, const uint16_t *codebooks,
                        const uint16_t *scales, const uint16_t *x, const uint16_t *gy, int T,
                        float *grad_scales, float *grad_codebooks, void *workspace,
                        size_t workspace_bytes, aq_stream_t stream);

/*
 * Measurement aid, not part of the product path: the codeword-read ceiling
 * of the 1x16 decode-time product.  A 1x16 layer decodes each code by
 * reading its 16-byte codeword from the 1 MiB codebook (the paper's 1x16
 * scheme: one codebook of 2^16 vectors of 8 weights); at decode batch
 * sizes these random reads, not HBM, bound aq_gemv.  aq_gather_probe
 * issues the same reads and nothing else, one per code:
 *   mode 0  from L2 into shared memory with cp.async, as aq_gemv's
 *           decoders do (two CTAs per SM, three stages in flight);
 *   mode 1  from the codebook split over the shared memory of 8-CTA
 *           thread-block clusters (128 KiB per CTA, loaded once per call)
 *           with distributed shared-memory loads;
 *   mode 2  into registers through L1 (ld.global.nc), as aq_gemv's batch-1
 *           1x16 path does (three CTAs of 256 threads per SM);
 *   mode 4  the codebook sliced over the shared memory of 8-CTA clusters
 *           (128 KiB per CTA, loaded once per call), the work moved to the
 *           slice: every CTA of a cluster reads the cluster's codes and
 *           reads, from its own shared memory, the codewords of the codes
 *           whose top 3 bits name its slice;
 *   mode 3  no codeword at all: `codes` itself is read once as a stream of
 *           16-byte loads (L1 bypassed, four CTAs of 256 threads per SM),
 *           the read-only HBM bandwidth when the array is much larger
 *           than L2 (a cross-check of the copy bandwidth the HBM roofline
 *           uses).  `codebook` is not read and may be NULL; the checksum
 *           XOR is then that of the codes' 32-bit words.
 *   codebook  [65536][8] binary16, device, 16-byte aligned (modes 0-2, 4),
 *   codes     n 16-bit codes, device, 16-byte aligned, n a multiple of 8
 *             (a 1x16 layer's packed codes are such an array),
 *   sink      device, >= aq_gather_probe_sink_bytes(mode) bytes, 16-byte
 *             aligned: receives 16-byte checksums, one per thread (the XOR
 *             of every 32-bit word it read); the XOR of all of them equals
 *             the XOR of codebook[codes[i]] over every i, if the sink was
 *             zero-filled first (threads without codes write zeros).
 * Asynchronous on `stream`, launched with programmatic stream
 * serialisation like aq_gemv, so back-to-back calls overlap the same way.
 * AQ_ERR_INVALID_ARG for another mode, null pointers, n = 0 or n not a
 * multiple of 8 (aq_gather_probe_sink_bytes returns 0 for another mode);
 * AQ_ERR_MISALIGNED for a pointer off a 16-byte boundary.
 */
size_t aq_gather_probe_sink_bytes(int mode);
aq_status aq_gather_probe(const uint16_t *codebook, const uint16_t *codes, size_t n, int mode, void *sink,
                          aq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AQ_B200_H */
