/*
 * entropack.h -- C ABI of the B200 lattice-rANS weight codec.
 *
 * The codec follows the EntroPack method: rows are normalised by their RMS and split into
 * 8-vectors, each vector is replaced by its nearest point of a scaled E8 lattice, the point is
 * stored as a coset bit plus eight integer fields, the fields are rANS-coded in independently
 * decodable tiles, and decoding rebuilds the weights on the GPU in one fused kernel.  Sources,
 * by page title and section: "EntroPack: Fast and Accurate Entropy-Coded Weight Compression at
 * Arbitrary Bitrates" (arXiv abstract); "EntroPack lattice compression" (documentation page
 * Principles / Lattice-rANS), sections "Lattice quantization and integer fields", "Rate
 * selection and refinement", "Encoding and reconstruction" and "Usage".
 *
 * Conventions (all calls):
 *   - Every int-returning call returns EP_OK (0) or a negative ep_status; a message describing
 *     the last failure on the calling thread is available from ep_last_error().
 *   - Pointers are plain host or device addresses; sizes are element or byte counts as stated.
 *     The header needs no CUDA include: a CUDA stream is passed as `void*` (a cudaStream_t;
 *     NULL means the legacy default stream).
 *   - Tensors are owned by the caller; blobs are owned by the library and released with
 *     ep_blob_free().
 */
#ifndef ENTROPACK_H
#define ENTROPACK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element containers.  By default a tensor is restored in the element type it was compressed
 * from ("EntroPack lattice compression", opening paragraph); the abstract names BF16, FP16, FP8
 * and INT8 containers.  FP32 is accepted as an extra container. */
typedef enum {
    EP_BF16 = 1,
    EP_FP16 = 2,
    EP_FP8_E4M3 = 3,  /* OCP E4M3 (bias 7, no infinities); outputs saturate to +-448 */
    EP_F32 = 4,
    EP_INT8 = 5       /* two's complement integers; outputs round to nearest (ties to even) and
                         saturate to [-128, 127] */
} ep_dtype;

typedef enum {
    EP_OK = 0,
    EP_ERR_ARG = -1,      /* NULL pointer, bad stride, unknown device                       */
    EP_ERR_DTYPE = -2,    /* unsupported container                                           */
    EP_ERR_SHAPE = -3,    /* empty tensor, or output shape differs from the blob's          */
    EP_ERR_RANGE = -4,    /* target bpp outside [0.001, 11] or not finite; non-finite weight */
    EP_ERR_CORRUPT = -5,  /* blob bytes fail validation, or the GPU decode found them broken */
    EP_ERR_CUDA = -6,     /* a CUDA runtime call failed (message in ep_last_error)           */
    EP_ERR_OOM = -7       /* host or device allocation failed                                */
} ep_status;

/* A 2-D tensor view.  Element (r, c) lives at data + (r * row_stride + c) * element size. */
typedef struct {
    void* data;
    int device;          /* -1: host memory; >= 0: CUDA device ordinal                          */
    int dtype;           /* ep_dtype                                                            */
    int64_t rows;
    int64_t cols;
    int64_t row_stride;  /* elements between consecutive rows, >= cols                         */
} ep_tensor;

/* Optional encoder settings (ep_compress uses all defaults). */
typedef struct {
    int steps_per_tile;  /* S in [1, 1024]: tile = 32*S vectors; 0 = clamp(next_pow2(ceil(128/bpp)), 16, 1024) */
    int num_threads;     /* host encoder threads; 0 = all hardware threads                       */
    double scale;        /* > 0: use this lattice scale instead of searching for one             */
    int rd_refine;       /* nonzero: per-row rate-distortion refinement ("Rate selection and
                            refinement": optional, off by default) -- every row picks one of five
                            resolutions s * 2^(k/2), k in {0, -1, 1, -2, 2}, by a Lagrangian
                            choice under the storage budget, in three rounds that rebuild the
                            probability tables; the decode format does not change           */
    int host_encoder;    /* nonzero: encode a device tensor on the host (it is copied there first);
                            by default a device tensor is encoded on its GPU -- the same bytes --
                            except with rd_refine, which runs on the host                    */
    int prob_bits;       /* frequency totals M = 2^prob_bits: 12 (the format's fixed choice, also
                            selected by 0) or 10 (a faster decode at a rate cost below 0.5% of the
                            coded bits); anything else is EP_ERR_ARG                          */
} ep_options;

typedef struct ep_blob ep_blob;

/* Header fields of a blob. */
typedef struct {
    int64_t rows, cols;
    int dtype;           /* input container recorded at compression */
    int steps_per_tile;  /* S */
    int64_t n_tiles;
    int64_t n_vectors;   /* rows * ceil(cols / 8) */
    double scale;        /* the shared lattice scale s chosen by the rate search */
    uint64_t bytes;      /* stored bytes, including all metadata */
    int prob_bits;       /* frequency totals 2^prob_bits (12 or 10) */
} ep_blob_info;

/*
 * Compress a 2-D tensor to a target rate ("EntroPack lattice compression": the opening paragraph
 * admits any finite rate from 0.001 to 11 bits per element, fractional ones included; sections
 * "Lattice quantization and integer fields" and "Rate selection and refinement").
 *   in          tensor to compress, host or device memory, any ep_dtype; rows, cols >= 1.
 *               Device tensors are copied to the host first (the encoder runs on the host).
 *   target_bpp  requested stored bits per element, finite, in [0.001, 11].
 *   out         receives a new blob (free with ep_blob_free).
 * Synchronous.  Errors: EP_ERR_ARG, EP_ERR_DTYPE, EP_ERR_SHAPE (empty), EP_ERR_RANGE,
 * EP_ERR_CUDA, EP_ERR_OOM.  Deterministic: the same input and settings give the same bytes.
 */
int ep_compress(const ep_tensor* in, double target_bpp, ep_blob** out);

/* ep_compress with explicit encoder settings (opt may be NULL for the defaults). */
int ep_compress_ex(const ep_tensor* in, double target_bpp, const ep_options* opt, ep_blob** out);

/*
 * Decompress into `out` ("EntroPack lattice compression", section "Encoding and
 * reconstruction": one fused GPU operation turns the coded fields back into lattice points,
 * multiplies them by the row scales and returns a tensor shaped and typed like the original).
 *   b       blob.
 *   out     rows x cols equal to the blob's; dtype any ep_dtype (the blob's own by convention).
 *           Device output (out->device >= 0, must be the calling thread's current device): one
 *           kernel launch on `stream`, asynchronous.  The first call on a device copies the
 *           blob to that device (it allocates and synchronises once; do that before any stream
 *           capture).  Later calls allocate nothing and do not synchronise.
 *           Host output (out->device == -1): end-to-end path on the current device -- copies the
 *           blob bytes host->device, decodes into a blob-owned device buffer, copies the result
 *           device->host into out->data, and returns when every row is there.  Blobs with 8 MB
 *           of output or more go in up to 8 chunks of whole rows: uploads and decodes run on
 *           `stream`, downloads on a copy-back stream the library keeps per device, so one
 *           chunk's download overlaps the next chunk's upload and decode (page-locked host
 *           memory lets the copies overlap; pageable memory works, slower).
 *   stream  cudaStream_t as void*.
 * Errors found on the GPU (corrupt tiles) are not returned here: read them with
 * ep_decode_status().  Returns EP_ERR_ARG, EP_ERR_SHAPE, EP_ERR_DTYPE, EP_ERR_CUDA, EP_ERR_OOM.
 * Not thread-safe for concurrent first calls on the same blob and device, nor for concurrent
 * host-output calls on the same blob (they share its staging buffers).
 */
int ep_decompress(const ep_blob* b, const ep_tensor* out, void* stream);

/*
 * Decompress a set of blobs -- for example the linear layers of one transformer block, decoded
 * just before they are used -- in as few kernel launches as possible: one per 28 blobs that share a frequency-total width.  Each
 * blob is decoded exactly as ep_decompress would decode it (same arithmetic, bit-identical
 * results); the launch divides the GPU among the blobs in proportion to their tiles, so small
 * matrices that would each leave most SMs idle share the GPU instead.  (The pages motivate it:
 * the abstract names diffusion denoising and transformer prefill, where a whole block's weights
 * are decoded online; the documentation's "Encoding and reconstruction" makes every tile
 * independently decodable, which is what lets tiles of different blobs run side by side.)
 *   blobs   n blob handles.
 *   outs    n device tensors on the current device, outs[i] shaped like blobs[i]; all n with the
 *           same dtype.  Host outputs are not accepted.
 *   n       number of blobs; n == 0 does nothing.
 *   stream  cudaStream_t as void*; asynchronous like ep_decompress on device outputs.
 * The first call for a blob on a device copies it there (allocates and synchronises once).  A
 * launch's table layout and CTA width follow from the tile count and largest tile of the blobs it
 * holds, so a set may need a blob's decode tables in a second layout: the first call that needs
 * it expands them (one allocation and one synchronisation per blob, device and layout); repeat
 * the call once before any stream capture.
 * Corrupt tiles are reported per blob by ep_decode_status().  Returns EP_ERR_ARG, EP_ERR_SHAPE,
 * EP_ERR_DTYPE, EP_ERR_CUDA, EP_ERR_OOM; nothing is launched when an argument is invalid.
 */
int ep_decompress_group(const ep_blob* const* blobs, const ep_tensor* outs, int n, void* stream);

/*
 * Decompress into the FP8 container with a per-row scale (the arXiv abstract lists FP8 among the
 * containers and keeps the stored bitrate apart from the restored precision).  Row r is written
 * as an E4M3 payload normalised to the format's range plus one fp32 scale sigma_r, so that
 * sigma_r * payload restores alpha_r * y:
 *   payload[r][c] = E4M3(RNE_fp32(y * g_r)), round to nearest even, saturating at +-448, with
 *                   g_r = RNE_fp32(896 / m_r) carrying alpha_r's sign (0 when m_r = 0 or
 *                   alpha_r = 0) and m_r the row's largest |2 y| (stored in the blob), so every
 *                   nonzero row reaches +-448;
 *   row_scale[r]  = RNE_fp32(|alpha_r| * m_r / 896) = rowmax |alpha_r * y| / 448.
 * Unlike the plain E4M3 container, small weights keep E4M3's relative precision instead of
 * falling into its subnormal range.
 *   b          blob.
 *   out        dtype EP_FP8_E4M3, rows x cols of the blob.  Device output (out->device >= 0,
 *              the current device): one fused kernel launch on `stream`, asynchronous; the first
 *              call on a device copies the blob there (allocates and synchronises once).  Host
 *              output (out->device == -1): the end-to-end path of ep_decompress -- upload, decode
 *              into blob-owned buffers, copy payload and scales back (in chunks of whole rows
 *              like ep_decompress), return when both are there.
 *   row_scale  rows floats (4-byte aligned), written: device memory on the current device for a
 *              device output, host memory for a host output.
 *   stream     cudaStream_t as void*.
 * Corrupt tiles are reported by ep_decode_status().  Returns EP_ERR_ARG (NULL pointers,
 * misaligned row_scale, other-device output), EP_ERR_DTYPE (output not E4M3), EP_ERR_SHAPE,
 * EP_ERR_CUDA, EP_ERR_OOM.
 */
int ep_decompress_fp8_rowscaled(const ep_blob* b, const ep_tensor* out, float* row_scale, void* stream);

/* Stored bits per element: 8 * (stored bytes including metadata) / (rows * cols)
 * ("EntroPack lattice compression", section "Encoding and reconstruction": the reported rate
 * counts every stored byte, metadata included, as bits per element).  Returns -1.0 for a NULL
 * blob. */
double ep_actual_bpp(const ep_blob* b);

/* Header fields of the blob. */
int ep_get_info(const ep_blob* b, ep_blob_info* info);

/* A view of the serialised bytes, valid until ep_blob_free(b). */
int ep_blob_to_bytes(const ep_blob* b, const uint8_t** data, size_t* n);

/* Copy and validate serialised bytes (header, sections, tables, tile offsets) into a new blob.
 * Returns EP_ERR_CORRUPT with a reason when the bytes are not a valid blob. */
int ep_blob_from_bytes(const uint8_t* data, size_t n, ep_blob** out);

/* Copy the blob to `device` now (otherwise the first ep_decompress does it), on `stream`,
 * and wait for the copy.  Lets a caller keep allocation out of a timed or captured region. */
int ep_blob_prepare(ep_blob* b, int device, void* stream);

/* Synchronise `stream`, then read and clear the blob's device status word on the current
 * device.  Returns EP_OK when every decode since the last call found consistent tiles, else
 * EP_ERR_CORRUPT with the failing checks in ep_last_error() (tile overrun, final rANS state
 * not 2^16, unused words, bad tile extent, bulk-copy wait limit). */
int ep_decode_status(const ep_blob* b, void* stream);

/* The kernel variant ep_decompress uses for this blob on the current device: the layout of the
 * decode tables in shared memory (10: 10-bit totals, one packed word per slot; 12, 13, 14: 12-bit
 * totals, with 0, 3 or 4 of a vector's 8 symbols read in one lookup and the rest in two) and the
 * CTA width in warps (16, 20, 24 or 32).  Both follow from the blob's tile count, its largest
 * tile and the device's SM count; no decode is launched.  A diagnostic for tests and profiles:
 * the method itself has no counterpart.  Returns EP_ERR_ARG (NULL pointer), EP_ERR_CUDA. */
int ep_decode_shape(const ep_blob* b, int* layout, int* warps);

/* Test hook: decode the fields of every vector into device memory `fields` (int16, n_vectors
 * x 9: column 0 the coset bit, columns 1..8 the fields f1..f8), asynchronously on `stream`.
 * Same kernel as ep_decompress up to the field inversion. */
int ep_decode_fields(const ep_blob* b, int16_t* fields, void* stream);

/*
 * Decode like ep_decompress, but allocate nothing -- no cudaMalloc, no host or device heap
 * allocation by the library.  (The method's pages have no counterpart: this is an interface for
 * callers that cannot let a library allocate GPU memory -- an inference runtime that plans all
 * device memory ahead of time in its own arena, or code running where allocation is forbidden or
 * would synchronise the device.)
 *   b                  blob handle; only its parsed header is used (its host bytes are not read).
 *   device_blob        the blob's serialised bytes (exactly those of ep_blob_to_bytes(b)) already
 *                      in device memory on the current device, owned by the caller, 16-byte
 *                      aligned.
 *   device_blob_bytes  size of the caller's device buffer; EP_ERR_ARG if it is smaller than the
 *                      blob.  The kernel reads nothing beyond the blob's size, and it checks
 *                      every tile's extent against the stream section before reading it, so a
 *                      stale or different copy is reported as corrupt rather than read outside
 *                      the buffer.
 *   out                device output on the current device, as for ep_decompress.
 *   stream             cudaStream_t as void*.
 *   wait               0: return after the launch (asynchronous; the kernel's corruption checks
 *                      are not reported, and ep_decode_status does not see them -- it reads the
 *                      blob's own status word, not this path's); nonzero: synchronise `stream`
 *                      and return EP_ERR_CORRUPT if the decode found a corrupt tile.
 * The decode kernel's scratch -- one 4-byte status word -- lives in a fixed 256-byte array of
 * device memory inside this library (64 words; every GPU that loads the library keeps it until
 * the process exits).  Each call clears the word it uses; a call whose scratch need exceeded the
 * array would be rejected with EP_ERR_ARG (no current launch needs more than one word).  All
 * calls share the array, which keeps the last call's contents, so calls that overlap on the GPU
 * (different streams, or several devices' host threads racing on one device) race on the status
 * word: serialise them or use ep_decompress.  The first call on each device looks up the array's
 * device address and sets the kernel's launch attributes; make that first call before any stream
 * capture.  The library allocates nothing, but the CUDA driver loads a kernel's code on its first
 * launch (lazy module loading, the driver's default), which can take device memory: a caller that
 * must see no allocation at all makes one call per output container and blob kind beforehand, or
 * runs with CUDA_MODULE_LOADING=EAGER.  Returns EP_ERR_ARG, EP_ERR_SHAPE, EP_ERR_DTYPE, EP_ERR_CUDA, EP_ERR_CORRUPT; messages
 * from this call never allocate.
 */
int ep_decompress_noalloc(const ep_blob* b, const void* device_blob, size_t device_blob_bytes, const ep_tensor* out,
                          void* stream, int wait);

/* Test hook for the bounded waits (the method's pages have no counterpart).  Launches the decode
 * kernel on the blob's device copy with every CTA waiting, for at most `wait_spins` polls, on a
 * shared-memory barrier that expects 16 bytes no copy delivers; the wait gives up, the CTA
 * records "bulk-copy wait limit reached" in the blob's status word, waits for its real copies and
 * leaves.  Nothing is decoded or written.  ep_decode_status then returns EP_ERR_CORRUPT, and the
 * context stays usable.  Returns EP_ERR_ARG (NULL blob, zero limit), EP_ERR_CUDA, EP_ERR_OOM. */
int ep_decode_wait_probe(const ep_blob* b, uint32_t wait_spins, void* stream);

/* Release a blob, its host bytes and any device copies (synchronises those devices). */
void ep_blob_free(ep_blob* b);

/* Message for the last failure on the calling thread ("" if none). */
const char* ep_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ENTROPACK_H */
