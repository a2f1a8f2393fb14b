/*
 * entropack.h -- C ABI of the EntroPack codec for B200 (sm_100a).
 *
 * EntroPack ("EntroPack: Fast and Accurate Entropy-Coded Weight Compression at
 * Arbitrary Bitrates") stores a weight matrix as independently decodable rANS
 * tiles of coset-conditioned E8-lattice fields, one FP32 reconstruction scale
 * per row, and seventeen frequency tables (§3.6 "Stored representation").
 * This library offers:
 *   ep_encode_tensor  -- the CPU packer (§3.1 pipeline, §3.4 scale search,
 *                        §3.5 refit, §3.6 tiles; App. C.1, C.3), threaded;
 *   ep_decode_tensor  -- the fused GPU reconstruction (Fig. 2b; §3.6: a warp
 *                        per tile, a lane per interleaved state; App. C.3),
 *                        stream-ordered, one kernel launch per call;
 * and, declared below with their own notes: the GPU encoder, the same decode
 * without a library allocation, prepared tables, batches of tensors (on all SMs
 * or a given number), and the product with 1 to 8 tokens taken inside the
 * decode (ep_decode_gemv).
 *
 * Stored representation (all little-endian; the packer writes it, the decoder
 * reads it):
 *   payload      uint16 words of all tiles, concatenated.
 *   tile_index   uint32[33*T + 1]: for tile t, [33t] = payload offset of the
 *                tile (in 16-bit words), [33t+1+j] = terminal rANS state of
 *                lane j (j < 32); [33T] = final boundary offset = payload size.
 *                (App. C.3: J = 32 states and one 32-bit offset per tile.)
 *   freq_tables  48-byte header {u32 magic 0x314B5045 "EPK1", u32 version 1,
 *                u32 b, u32 V, u32 J = 32, u32 T, i64 rows, i64 cols,
 *                u32 ntables = 17, u32 flags = 0}, then 17 x {i32 min, u32 A},
 *                zero padding to a multiple of 16 bytes, then the uint16
 *                frequencies of every table in table order (A per table).
 *                Table 0 codes the coset bit c; table 1 + 2(k-1) + c codes field
 *                k (z1..z7, then m) of a vector in coset c (App. A.3).
 *   row_scales   float32[rows]: reconstruction scale of each row.
 * Vector g (8 consecutive weights of a row, g = row*nq + col/8, nq = ceil(cols/8):
 * a partial last vector of a row is padded with zeros) lies in tile g / V, on
 * lane (g mod V) mod 32, round (g mod V) / 32 (the lane interleave).
 */
#ifndef ENTROPACK_H
#define ENTROPACK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Output element types of the decoder. */
typedef enum {
    EP_BF16 = 0,        /* bfloat16, round to nearest even */
    EP_FP16 = 1,        /* IEEE binary16, round to nearest even, overflow to inf */
    EP_FP8_E4M3 = 2,    /* OCP FP8 E4M3 ("fn"), round to nearest even, saturating to +-448 */
    EP_INT8 = 3,        /* nearest-even integer, clamped to [-127, 127] */
    EP_FP32 = 4,        /* the FP32 product itself */
    EP_LATTICE_I32 = 5, /* int32 2y (twice the lattice coordinates), for verification */
    EP_UINT8 = 6        /* the UINT8 container with its offset: nearest-even integer, clamped to
                           [-128, 127], plus 128 (App. B, Table 6: unsigned integer inputs carry an
                           offset, which the codec removes before coding and adds back here) */
} ep_dtype;

typedef enum {
    EP_OK = 0,
    EP_EINVAL = 1,        /* a null pointer, a bad size, a misaligned buffer */
    EP_EUNSUPPORTED = 2,  /* an unknown dtype, a format variant the GPU does not decode */
    EP_EALPHABET = 3,     /* the packer could not fit the alphabets (should not happen) */
    EP_ECUDA = 4,         /* a CUDA runtime error at launch */
    EP_ECORRUPT = 5,      /* the device found an inconsistent stream or table header */
    EP_ENOMEM = 6         /* host allocation failed in the packer */
} ep_status;

/* Packer options; zero-initialise and set what you need. */
typedef struct {
    int prob_bits;            /* starting precision b in [9, 15]; 0: 11 for targets <= 7 bpp, else 12 (App. C.1) */
    int tile_vectors;         /* V; 0: max(32, floor(S/9)), S = 32768 / 16384 / 8192 / 4096 by target (Table 5) */
    int64_t sample_vectors;   /* rate-estimation sample; 0: 2^18 vectors of complete rows (App. C.1) */
    int search_steps;         /* geometric bisection steps; 0: 12 (App. C.1) */
    uint64_t seed;            /* sample seed; 0: derived from the shape */
    int has_container_scales; /* 1: count 4 bytes per row of FP8/INT8 container scales in the rate */
    int num_threads;          /* 0: all hardware threads */
    int rdo_candidates;       /* per-row rate-distortion refinement (§3.5, App. C.2): K candidate
                                 scales per row (0 or 1: off, the default, as in the paper's results) */
    int rdo_sweeps;           /* its allocation sweeps; 0: 1 */
} ep_encode_opts;

/* The packer's output; host memory owned by the library, freed by ep_free_blob. */
typedef struct {
    int64_t rows, cols;
    int b;                 /* probability precision, M = 2^b */
    int V;                 /* vectors per tile */
    int J;                 /* 32 */
    int ntiles;            /* T */
    uint16_t* payload;     /* payload_words words, followed by zero words up to a multiple of 8 */
    size_t payload_words;  /* the stored payload (= tile_index[33T]) */
    size_t payload_alloc_words; /* payload_words rounded up to a multiple of 8 */
    uint32_t* tile_index;  /* 33*T + 1 words */
    uint8_t* freq_tables;  /* freq_bytes bytes */
    size_t freq_bytes;
    float* row_scales;     /* rows floats */
    double s;              /* selected quantisation scale */
    double stored_bpp;     /* 8 * stored_bytes / (rows*cols)  ([paper] §4.1 "Metrics") */
    int64_t stored_bytes;  /* payload + tile metadata + tables + row scales (+ container scales) */
} ep_blob;

/*
 * ep_encode_tensor -- compress W (host, row-major float32 [rows, cols], the
 * container's values) to about target_bpp stored bits per weight.
 * Follows §3.1: row normalisation, sampled-row scale search (§3.4, App. C.1),
 * E8 quantisation, row-scale refit (§3.5), optional per-row refinement (§3.5,
 * App. C.2: K candidate scales per row, allocated under the baseline's code
 * length; memory grows by K x 36 bytes per vector), seventeen tables and tiled
 * interleaved rANS (§3.6, App. C.3).  Runs on the host with num_threads threads.
 * opts may be NULL.  On EP_OK *out holds a new blob (free with ep_free_blob).
 * Errors: EP_EINVAL (null W/out, rows or cols <= 0, target_bpp <= 0, b out of
 * [9, 15]), EP_EALPHABET, EP_ENOMEM.  A width that is not a multiple of 8 pads every
 * row with zeros to whole vectors (the normaliser, refit and rate use the real
 * entries only); the decoder drops the padding.
 */
ep_status ep_encode_tensor(const float* W, int64_t rows, int64_t cols, double target_bpp,
                           const ep_encode_opts* opts, ep_blob** out);

/*
 * ep_encode_tensor_gpu -- the packer of ep_encode_tensor with its full-tensor
 * stages on the GPU: row normalisation, the quantisation of the sampled rows
 * for every step of the scale search and of the whole tensor, the symbol
 * counts, the row-scale refit and the tiled rANS (one warp per tile).  The
 * search's decisions, the table normalisation, the per-row refinement's lambda
 * bisection (App. C.2; the candidates are quantised, refitted and priced on the
 * GPU) and the header stay on the host.
 * The blob is byte for byte the one ep_encode_tensor returns for the same
 * matrix and options: every floating-point step is the host's operation in the
 * host's order, without multiply-add contraction, and the estimates' bits come
 * from exact counts (paper §3.1 pipeline; §3.4, §3.5, §3.6, App. C.1, C.3).
 *   stream  cudaStream_t to launch on (the call synchronises it several times).
 *   W       device, float32 [rows, cols] row-major, 4-byte aligned; not modified.  A
 *           pointer that is not device memory of the current device (or managed
 *           memory) is refused with EP_EINVAL before any launch.
 *   opts    as ep_encode_tensor (num_threads is ignored).
 * Scratch (about 54 bytes per vector of eight weights, more with the per-row
 * refinement: 36 per vector per candidate) comes in stream order from a memory
 * pool the library creates per device, which keeps up to 1 GiB between calls
 * and returns the rest to the device.  On EP_OK *out holds a host blob
 * (free with ep_free_blob).  Errors: EP_EINVAL, EP_EUNSUPPORTED, EP_EALPHABET,
 * EP_ENOMEM, EP_ECUDA.
 */
ep_status ep_encode_tensor_gpu(void* stream, const float* W, int64_t rows, int64_t cols, double target_bpp,
                               const ep_encode_opts* opts, ep_blob** out);

/*
 * A compressed tensor in device memory, as ep_encode_tensor_gpu_device returns
 * it: the four stored arrays of ep_blob (the same bytes), each in its own
 * cudaMalloc allocation that the struct owns (free with ep_free_device_blob).
 * The buffers meet ep_decode_tensor's alignment and padding rules.
 */
typedef struct {
    int64_t rows, cols;
    int b, V, ntiles;
    uint64_t payload_words;      /* words of payload (the last tile's end offset) */
    size_t payload_alloc_words;  /* payload_words rounded up to 8 (the tail is zero) */
    size_t freq_bytes;
    uint16_t* payload;           /* device */
    uint32_t* tile_index;        /* device, 33 * ntiles + 1 words */
    uint8_t* freq_tables;        /* device, freq_bytes */
    float* row_scales;           /* device, rows */
    double s, stored_bpp;
    int64_t stored_bytes;
} ep_device_blob;

/*
 * ep_encode_tensor_gpu_device -- ep_encode_tensor_gpu with the compressed
 * tensor left in device memory (no copy to the host): for a model whose
 * weights are loaded to the GPU and compressed there.  W is float32 (w_is_bf16
 * = 0, 4-byte aligned) or bfloat16 (w_is_bf16 = 1, 2-byte aligned; widened to
 * float32 exactly on the GPU, so the bytes are those of the packer on the
 * widened matrix).  *out receives the arrays in new device allocations
 * (cudaMalloc); the scratch comes from the same pool as ep_encode_tensor_gpu's
 * (a bfloat16 matrix adds 4 bytes per weight).  Errors as ep_encode_tensor_gpu
 * (on an error *out is left empty).
 */
ep_status ep_encode_tensor_gpu_device(void* stream, const void* W, int w_is_bf16, int64_t rows, int64_t cols,
                                      double target_bpp, const ep_encode_opts* opts, ep_device_blob* out);

/* Free the device arrays of an ep_device_blob and clear it (NULL and empty blobs are allowed). */
void ep_free_device_blob(ep_device_blob* blob);

/* Free a blob returned by ep_encode_tensor or ep_encode_tensor_gpu (NULL is allowed). */
void ep_free_blob(ep_blob* blob);

/*
 * ep_decode_tensor -- reconstruct the dense [rows, cols] matrix on the GPU
 * (Fig. 2b: symbol decode, lattice reconstruction, row rescale, dtype
 * conversion fused in one pass; App. C.3 tile layout).
 *   stream       cudaStream_t to launch on (NULL: the legacy default stream).
 *   tiles        device, the payload; 16-byte aligned; the buffer must be
 *                readable up to the final offset rounded up to a multiple of 8
 *                words (the packer's payload_alloc_words).
 *   tile_index   device, uint32[33*T + 1], 4-byte aligned.  Its last word, the
 *                final payload offset, is trusted: it must not exceed the words the
 *                tiles buffer holds (the signature carries no payload length, so
 *                the kernel bounds every payload read by that word and by the
 *                tile offsets, which it checks against it).
 *   freq_tables  device, the table header and frequencies, 16-byte aligned.  The
 *                buffer must hold the frequencies its header describes.
 *   row_scales   device, float32[rows].
 *   rows, cols   the matrix shape; must match the header.
 *   out_dtype    one of ep_dtype.
 *   out          device, rows*cols elements of out_dtype, row-major, 16-byte aligned
 *                (the padding of rows whose width is not a multiple of 8 is not
 *                written; such rows are written element by element).
 * All buffers belong to the caller.  The library keeps one 128 KB workspace
 * per device (allocated with cudaMalloc and zeroed on the first call on that
 * device, so make the first call before any stream capture); every CTA writes
 * its share of the decode lookup table there and reads the whole table back
 * (a table built once across the grid costs less than one built in every
 * CTA).  Decodes on one device are ordered through that workspace: a call
 * waits on the GPU for the previous call, whatever stream it ran on (not
 * applied while the stream is being captured), so per-call decodes on two
 * streams run one after the other; prepared-table and batched decodes use no
 * workspace and may overlap.
 * The call is asynchronous: it validates the arguments on the host and makes
 * one cooperative launch on the stream (one CTA per SM).  Argument errors
 * return at once (EP_EINVAL, EP_EUNSUPPORTED), launch errors as EP_ECUDA.  The
 * stream itself is checked on the device without trapping: a corrupt payload,
 * state, offset or table raises a device-side status word that
 * ep_decode_status reads.  Outputs of a corrupt tile are unspecified; no access
 * leaves the buffers described above.
 */
ep_status ep_decode_tensor(void* stream, const uint16_t* tiles, const uint32_t* tile_index,
                           const uint8_t* freq_tables, const float* row_scales, int64_t rows,
                           int64_t cols, ep_dtype out_dtype, void* out);

/*
 * ep_decode_tensor_noalloc -- the same decode as ep_decode_tensor, for callers
 * that cannot allocate device memory: code whose memory is owned by another
 * allocator (a framework's caching allocator, a memory budget fixed at start-up),
 * code that must not take the implicit device synchronisation of cudaMalloc
 * (latency-critical serving loops), and code that runs where allocation is not
 * permitted.  There is no counterpart in the EntroPack paper; the arguments,
 * alignment rules, output and status reporting are those of ep_decode_tensor.
 * Its scratch (the decode lookup-table image and 32 bytes of grid-barrier state,
 * 131,104 bytes in all: enough for any stream with b <= 15) lives in a
 * fixed-size device array inside the library; every GPU that loads the library
 * keeps that array until the process exits.  The call allocates and frees
 * nothing: on the first call on a device (which must come before any stream
 * capture) it looks up the array's device address; each call then clears the
 * barrier words with cudaMemsetAsync and makes one cooperative launch.
 * Every call shares the array and it keeps the last call's contents, so calls
 * whose executions overlap on the GPU (for instance on two streams) race on it
 * and must be ordered by the caller.  Tensors of 2^31 vectors (of 8 weights) or
 * more are rejected with EP_EINVAL, like every other size error.
 */
ep_status ep_decode_tensor_noalloc(void* stream, const uint16_t* tiles, const uint32_t* tile_index,
                                   const uint8_t* freq_tables, const float* row_scales, int64_t rows,
                                   int64_t cols, ep_dtype out_dtype, void* out);

/*
 * Size in bytes of a prepared decode table: the lookup-table image (128 KiB,
 * enough for any stream with b <= 15) and a 32-byte trailer.
 */
#define EP_LUT_BYTES 131104

/*
 * ep_decode_prepare -- build a tensor's decode lookup table once, into a
 * caller buffer that later decodes of the same tensor read instead of building
 * it again.  The tables map the low b bits of a rANS state to a symbol and its
 * frequency interval (App. C.3, "Decoder lookup tables": the tables sit in
 * shared memory or in packed global memory); they depend only on freq_tables,
 * so a weight that is decoded many times (every denoising step, every prefill)
 * can keep them beside its compressed bytes.
 *   stream       cudaStream_t to launch on.
 *   freq_tables  device, the tensor's table header and frequencies (16-byte aligned).
 *   rows, cols   the matrix shape; must match the header.
 *   lut          device, lut_bytes >= EP_LUT_BYTES, 16-byte aligned, owned by the
 *                caller; written by this call (one memset of the trailer and one
 *                launch on `stream`), read by ep_decode_tensor_prepared.
 * Argument errors return at once (EP_EINVAL); launch errors as EP_ECUDA.  An
 * invalid header or tables that do not sum to 2^b raise the device status word
 * (ep_decode_status); a decode with that table raises it again.
 */
ep_status ep_decode_prepare(void* stream, const uint8_t* freq_tables, int64_t rows, int64_t cols, void* lut,
                            size_t lut_bytes);

/*
 * ep_decode_tensor_prepared -- ep_decode_tensor with the lookup table that
 * ep_decode_prepare built from the same freq_tables.  The arguments, alignment
 * rules, output and status reporting are those of ep_decode_tensor, plus
 *   lut, lut_bytes  the prepared table (device, >= EP_LUT_BYTES, 16-byte aligned;
 *                   read only, so any number of decodes may share it at once).
 * The call uses no library workspace and no grid-wide barrier: it makes one
 * ordinary launch on the stream (one CTA per SM), so decodes on different
 * streams may run at the same time and nothing orders them but their streams.
 * The launch allows programmatic dependent launch: the kernel may be scheduled
 * while the kernel ahead of it in the stream is ending, and it waits for that
 * kernel to complete before its first global-memory access.
 * A table whose layout does not match this tensor's header (b, LUT format, or
 * any table's minimum or alphabet size), or a buffer ep_decode_prepare did not
 * write, raises EP_ECORRUPT in the status word and nothing is decoded.  A table
 * prepared from tables with the same layout but other frequencies is not
 * detected: the output is then unspecified, and every access stays in bounds.
 */
ep_status ep_decode_tensor_prepared(void* stream, const uint16_t* tiles, const uint32_t* tile_index,
                                    const uint8_t* freq_tables, const float* row_scales, const void* lut,
                                    size_t lut_bytes, int64_t rows, int64_t cols, ep_dtype out_dtype,
                                    void* out);

/*
 * ep_decode_gemv -- a linear layer on a few tokens with the weight decoded inside the product
 * (the on-demand reconstruction of paper §4.3 and Fig. 5, for the decode-bound case of
 * small token counts): y = x W^T, where W [rows, cols] is the tensor's decoded weight in
 * BF16 (the values ep_decode_tensor writes for EP_BF16) and x holds BF16 activations: the
 * numerics of a BF16 GEMM (exact products, float32 accumulation).  Every lane rounds the
 * eight weights it has just reconstructed to BF16 and multiplies them by the tokens' eight
 * activations of those columns with float32 multiply-adds, accumulating per row; the weight
 * is never written to memory.
 *   tiles .. cols   as ep_decode_tensor (cols must be a multiple of 8: else EP_EUNSUPPORTED).
 *   lut, lut_bytes  a table ep_decode_prepare built for this tensor (then the call uses no
 *                   workspace and launches as ep_decode_tensor_prepared), or NULL (the table
 *                   is built per call in the workspace, as ep_decode_tensor).
 *   x               device, BF16 bits [ntok, cols] row-major, 16-byte aligned; read only.
 *   ntok            1, 2, 4 or 8 (else EP_EUNSUPPORTED).
 *   y               device, float32 [ntok, rows] row-major, 16-byte aligned; overwritten: it
 *                   is zeroed first (with a prepared table by a memset on the stream, else by
 *                   the kernel before its grid barrier), then the partial sums of each row are
 *                   added by atomic adds, so the order of the float32 additions is unspecified
 *                   (the result lies within the float32 dot-product bound of the exact
 *                   product).  After a stream error its contents are unspecified.
 * Asynchronous on `stream`; argument errors as ep_decode_tensor; stream errors raise the
 * status word that ep_decode_status reads.
 */
ep_status ep_decode_gemv(void* stream, const uint16_t* tiles, const uint32_t* tile_index, const uint8_t* freq_tables,
                         const float* row_scales, const void* lut, size_t lut_bytes, int64_t rows, int64_t cols,
                         const void* x, int ntok, float* y);

/*
 * Batched decode: several tensors in one launch.  A layer-by-layer decode leaves
 * most of the GPU idle on small tensors and on low rates (few tiles, each a long
 * sequential chain: at the pages' tile sizes a 3840x3840 weight has under two
 * tiles per warp scheduler); a batch shares the SMs out among its tensors, so
 * the tiles of all of them run side by side.  There is no counterpart in the
 * EntroPack paper; each tensor is decoded exactly as by ep_decode_tensor (one
 * warp per tile, the same tables and arithmetic), only the assignment of tiles
 * to SMs differs.
 *
 * ep_batch_item: one tensor of a batch; the pointers, shapes and alignment rules
 * of ep_decode_tensor_prepared, plus
 *   lut             its prepared table (ep_decode_prepare), EP_LUT_BYTES;
 *   ntiles, tile_vectors, prob_bits
 *                   T, V and b of its stream (the packer's blob fields).  They
 *                   only weigh the tensor when the SMs are shared out; the
 *                   decode itself takes T, V and b from the table header.
 */
typedef struct {
    const uint16_t* tiles;
    const uint32_t* tile_index;
    const uint8_t* freq_tables;
    const float* row_scales;
    const void* lut;
    int64_t rows, cols;
    int64_t ntiles, tile_vectors;
    int prob_bits;
    void* out;
} ep_batch_item;

typedef struct ep_batch ep_batch;

/*
 * ep_batch_create -- plan one launch that decodes items[0..n_items) into
 * out_dtype.  Every SM runs one CTA, which decodes a share of one tensor's
 * tiles; each tensor gets at least one SM and at most one per tile, the rest
 * going one by one to the tensor a simple cost model says finishes last
 * (ep_batch_apportion).  At most one tensor per SM (n_items <= the SM count,
 * else EP_EINVAL).  The plan (the items' pointers and shares, 80 bytes per SM)
 * is copied to a device buffer the handle owns (cudaMalloc + a synchronous
 * copy: create batches before any stream capture).  The items' buffers stay
 * the caller's and must outlive the handle.  Argument errors: EP_EINVAL,
 * EP_EUNSUPPORTED; CUDA errors: EP_ECUDA.  On success *out holds the handle.
 */
ep_status ep_batch_create(const ep_batch_item* items, int n_items, ep_dtype out_dtype, ep_batch** out);

/*
 * ep_batch_create_on -- ep_batch_create on num_ctas SMs instead of all of them
 * (num_ctas = 0: all; else n_items <= num_ctas <= the SM count, else
 * EP_EINVAL).  The launch has num_ctas CTAs, so the other SMs stay free for
 * kernels on other streams.  Each warp decodes one tile at a time as one
 * sequential chain, so a tensor whose tiles outnumber its CTAs' warps (24 per
 * CTA) takes more than one chain's time.  Same ownership and errors as
 * ep_batch_create.
 */
ep_status ep_batch_create_on(const ep_batch_item* items, int n_items, ep_dtype out_dtype, int num_ctas,
                             ep_batch** out);

/*
 * ep_decode_batch -- one launch on `stream` (an ordinary launch, one CTA per
 * SM, with programmatic dependent launch as ep_decode_tensor_prepared's) that
 * decodes every tensor of the batch into its `out`.  Outputs, status
 * reporting and the checks of each tensor's header and table are those of
 * ep_decode_tensor_prepared.  The current device must be the one the batch was
 * created on (else EP_EINVAL).  Capturable in a CUDA graph.
 */
ep_status ep_decode_batch(void* stream, const ep_batch* batch);

/* Free a batch handle (NULL is allowed); synchronises the device (cudaFree). */
void ep_batch_free(ep_batch* batch);

/*
 * ep_batch_apportion -- the host-only share-out ep_batch_create uses: counts[k]
 * SMs for tensor k, each in [1, ntiles[k]], together at most num_ctas (fewer
 * when the tensors have fewer tiles than that).  EP_EINVAL when n <= 0,
 * num_ctas < n, a pointer is NULL or a tensor has no tile.
 */
ep_status ep_batch_apportion(int n, const int64_t* ntiles, const int64_t* tile_vectors, const int* prob_bits,
                             int num_ctas, int* counts);

/*
 * ep_decode_status -- synchronise `stream`, read and clear the status word of
 * the current device: EP_OK, EP_ECORRUPT (an inconsistent stream or header),
 * or EP_EUNSUPPORTED (a header variant the GPU decoder does not handle).
 * The word is shared by every decode on the device since the last read.
 */
ep_status ep_decode_status(void* stream);

/* A static description of a status code. */
const char* ep_status_string(ep_status s);

#ifdef __cplusplus
}
#endif
#endif /* ENTROPACK_H */
