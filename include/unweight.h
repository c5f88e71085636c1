/*
 * unweight.h -- C ABI of libunweight: lossless BF16 weight compression with
 * the decode fused into the matrix product, for NVIDIA B200 (sm_100a).
 *
 * The method is the one described on the web page "Cloudflare推出Unweight無損壓縮
 * 系統，將LLM模型大小壓縮15-22%" (easyvibecoding.app):
 *   §BF16權重壓縮原理   each BF16 weight splits into a sign+mantissa byte, kept
 *                       as is, and an exponent byte; exponents are Huffman
 *                       coded or mapped to a 4-bit index into a per-matrix
 *                       palette of the 16 most frequent exponents; a 64-weight
 *                       row holding an exponent outside the palette is stored
 *                       verbatim.
 *   §四種執行管道       four pipelines: full decode + dense GEMM, exponent-only
 *                       decode + reconstructive GEMM, palette transcode +
 *                       reconstructive GEMM, direct palette GEMM.
 *   §重建矩陣乘法核心運作 the reconstructive GEMM rebuilds BF16 tiles in shared
 *                       memory and feeds them straight to the tensor cores.
 *   §解壓與運算資源共享  decoder and GEMM may share the GPU, split by SMs.
 *   §自動調優機制       an autotuner picks pipeline and SM split per projection
 *                       and batch size by measurement.
 *
 * Conventions for every call:
 *   - Pointers named *_dev / device buffers are device memory owned by the
 *     caller; the library never allocates device memory.  Host pointers are
 *     owned by the caller as well.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *     Calls are asynchronous on that stream unless stated otherwise.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns a status and launches nothing.
 *   - Device-detected problems (an undecodable stream, a bounded wait that
 *     expired) set a device status word; read it with uw_last_device_status.
 *   - Matrices are row-major.  W is [N, K] (output features x input features,
 *     the nn.Linear layout), X is [M, K], Y is [M, N].  BF16 values are passed
 *     as their 16-bit patterns (uint16_t).
 *   - K must be a positive multiple of 64 and N*K at most 2^31 - 256.
 */
#ifndef UNWEIGHT_H
#define UNWEIGHT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    UW_OK = 0,
    UW_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, misaligned pointer    */
    UW_ERR_SHAPE = 2,        /* K % 64 != 0, K < 64, N < 1, N*K too large     */
    UW_ERR_CORRUPT = 3,      /* serialized blob fails validation              */
    UW_ERR_UNSUPPORTED = 4,  /* pipeline needs a form the blob does not hold  */
    UW_ERR_WORKSPACE = 5,    /* buffer too small or misaligned                */
    UW_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed             */
    UW_ERR_TIMEOUT = 7,      /* a bounded device-side wait expired            */
    UW_ERR_DEVICE = 8        /* a device-side check failed (bad stream data)  */
} uw_status;

/* The four pipelines of §四種執行管道, a fifth that decodes the Huffman
 * stream inside the product (the pages could not fit the decode table beside
 * the Hopper matmul's buffers, §解壓與運算資源共享), and the autotuned
 * choice of §自動調優機制 (UW_PIPE_AUTO: the plan given in the options picks
 * the pipeline and matmul settings for this projection and batch size). */
typedef enum {
    UW_PIPE_AUTO = -1,           /* resolved through uw_gemm_opts.plan (see uw_plan_resolve)  */
    UW_PIPE_FULL = 0,            /* Huffman full decode -> BF16 W in workspace -> dense GEMM  */
    UW_PIPE_EXPONENT = 1,        /* Huffman exponent decode -> E in workspace -> reconstructive GEMM */
    UW_PIPE_TRANSCODE = 2,       /* Huffman -> 4-bit index plane in workspace -> reconstructive GEMM */
    UW_PIPE_DIRECT_PALETTE = 3,  /* reconstructive GEMM straight from the stored index plane */
    UW_PIPE_FUSED_HUFFMAN = 4    /* an addition to the four: the Huffman stream decoded inside the
                                    product itself (no decoded plane in HBM); CUDA cores, batches of
                                    up to 16 rows per pass (larger M: one pass per 16 rows); needs
                                    the Huffman form and K a multiple of 256 (else
                                    UW_ERR_UNSUPPORTED); variant, grid, split_k and sm_dec are
                                    ignored.  Its summation order differs from the other
                                    pipelines' (k ranges of 256-weight segments per warp, added in
                                    order), so it agrees with them within the GEMM tolerance, not
                                    bit for bit; it does not depend on the launch. */
} uw_pipeline;

/* Matmul variant: which kernel family computes the product. */
typedef enum {
    UW_VARIANT_AUTO = 0,     /* batch 1 on a projection with fewer than grid/2 tiles of 128 rows
                                runs the CUDA-core GEMV, everything else the tensor cores      */
    UW_VARIANT_TENSOR = 1,   /* tcgen05 tensor-core kernel at every batch size                 */
    UW_VARIANT_GEMV = 2      /* CUDA-core GEMV (batch 1 only; other batches: UW_ERR_UNSUPPORTED) */
} uw_variant;

/* Forms a compressed matrix may hold (bit mask). */
enum { UW_FORM_HUFFMAN = 1, UW_FORM_PALETTE = 2 };

/* Sections of a compressed matrix's device image. */
typedef enum {
    UW_SEC_SM = 0,        /* u8[N*K]  sign+mantissa bytes                          */
    UW_SEC_VBITS = 1,     /* u32[ceil(G/32)] verbatim flag per 64-weight group     */
    UW_SEC_VPRE = 2,      /* u32[ceil(G/32)] verbatim groups before word w         */
    UW_SEC_VEXP = 3,      /* u8[V*64] raw exponents of verbatim groups             */
    UW_SEC_VCOL = 4,      /* u32[(K/64)*4*ceil(N/128)] verbatim flags, by column   */
    UW_SEC_IDX = 5,       /* u8[N*K/2] 4-bit palette indices (palette form)        */
    UW_SEC_STREAM = 6,    /* u32[] Huffman stream, MSB first (Huffman form)        */
    UW_SEC_CHUNK_OFF = 7, /* u64[ceil(nseg/16)] bit offset of symbol 4096c         */
    UW_SEC_SEG_REL = 8,   /* u16[nseg] bit offset of symbol 256j minus chunk offset */
    UW_SEC_LUT = 9,       /* u32[4096] derived multi-symbol decode table (not serialized) */
    UW_NSECT = 10
} uw_section;

typedef struct uw_blob uw_blob;   /* opaque host handle of one compressed matrix */

typedef struct {
    int64_t N, K;             /* matrix shape                                         */
    int64_t G;                /* 64-weight groups = N*K/64                             */
    int64_t V;                /* verbatim groups                                       */
    int64_t nseg, nchunk;     /* 256-symbol segments, 16-segment chunks                */
    uint32_t forms;           /* UW_FORM_* held                                        */
    uint8_t palette[16];      /* exponent of each palette index                        */
    uint8_t code_len[16];     /* Huffman code length of each index (0 = unused)        */
    uint64_t freq[16];        /* symbol counts                                         */
    uint64_t hist[256];       /* exponent histogram                                    */
    uint64_t total_bits;      /* Huffman stream length                                 */
    uint64_t bytes_huffman_form;  /* sm + stream + offsets + verbatim store            */
    uint64_t bytes_palette_form;  /* sm + idx + verbatim store + vcol                  */
    uint64_t device_bytes;    /* size of the device image                              */
    double mean_code_len;     /* bits per weight of the Huffman stream                 */
    double exponent_entropy;  /* entropy of the exponent histogram, bits               */
    double palette_coverage;  /* share of weights whose exponent is in the palette     */
    uint64_t section_offset[UW_NSECT];  /* byte offset in the device image             */
    uint64_t section_bytes[UW_NSECT];   /* byte length (0 = absent)                    */
} uw_blob_info;

/* One autotuner decision (§自動調優機制): the configuration chosen for one
 * projection and one batch size. */
typedef struct {
    int32_t blob_index;      /* which projection (its index in the autotuner's blobs)     */
    int64_t M;               /* batch size                                                */
    int32_t pipeline;        /* chosen uw_pipeline (never UW_PIPE_AUTO)                   */
    int32_t variant;         /* chosen uw_variant                                         */
    int32_t sm_dec;          /* chosen decoder SM count (0: decode, then GEMM)            */
    int32_t grid;            /* chosen tensor-core CTA count (0: default rule)            */
    int32_t split_k;         /* chosen k ranges per output tile (0: default rule)         */
    double us;               /* measured time of this projection alone, microseconds      */
    double layer_us;         /* measured time of the whole sequence of projections        */
} uw_plan_entry;

typedef struct {
    int32_t pipeline;        /* uw_pipeline                                               */
    int32_t sm_dec;          /* >0: the Huffman decoder runs on sm_dec SMs beside the GEMM
                                in one launch (§解壓與運算資源共享); 0: decode, then GEMM */
    int32_t grid;            /* tensor-core GEMM CTAs; 0 = one per SM, or, when batch
                                tiles have 64+ rows and there are no more output tiles than
                                SMs, the largest whole multiple of the tile count that
                                fits.  With UW_VARIANT_AUTO it also decides whether batch 1
                                runs the CUDA-core GEMV (see uw_gemm)                      */
    int32_t out_f32;         /* 0: Y is BF16 (round to nearest even); 1: Y is float32      */
    int32_t variant;         /* uw_variant                                                 */
    int32_t split_k;         /* 0: grid decides; >0: every output tile is cut into split_k
                                k ranges (at most its k steps), one CTA each, grid ignored.
                                split_k >= 2 needs tiles * split_k <= SMs (else
                                UW_ERR_INVALID_ARG)                                        */
    int32_t stages;          /* 0: the deepest stage ring that fits; >= 2: at most this many */
    int32_t projection;      /* UW_PIPE_AUTO: the projection index looked up in `plan`     */
    const uw_plan_entry* plan;   /* UW_PIPE_AUTO: the autotuner's entries (host memory)    */
    int32_t plan_entries;
    void* workspace;         /* device, 256-byte aligned, any contents; a call owns it
                                until it completes (one workspace per stream)              */
    size_t workspace_bytes;
} uw_gemm_opts;

/* ---------------------------------------------------------------- misc */

/* Human-readable name of a status.  Never NULL. */
const char* uw_status_str(int status);

/* Library version (major*10000 + minor*100 + patch). */
int uw_version(void);

/* Synchronizes `stream`, then returns and clears the device status word of
 * the current device: UW_OK, UW_ERR_TIMEOUT or UW_ERR_DEVICE. */
uw_status uw_last_device_status(void* stream);

/* ---------------------------------------------------------------- compress
 * Load-time compression (§BF16權重壓縮原理; "模型載入時預轉", §四種執行管道).
 * Two steps so that the caller allocates the device image:
 *   1. uw_compress_query analyses W (histogram, palette, verbatim groups,
 *      Huffman code, segment offsets) and reports the image size;
 *   2. uw_compress_commit writes every section into the caller's buffer.
 * Both synchronize `stream`.  `scratch` is device memory of at least
 * uw_compress_scratch_bytes(N, K), 256-byte aligned, used only during these
 * calls.  W must stay unchanged between the two calls. */
uw_status uw_compress_scratch_bytes(int64_t N, int64_t K, size_t* bytes);

/* W_dev: device BF16 [N,K]; forms: UW_FORM_HUFFMAN | UW_FORM_PALETTE (nonzero).
 * On success *out is a new handle (free with uw_blob_free) and *dev_bytes the
 * size of the device image to allocate (256-byte aligned). */
uw_status uw_compress_query(const uint16_t* W_dev, int64_t N, int64_t K, uint32_t forms,
                            void* scratch, size_t scratch_bytes, void* stream,
                            uw_blob** out, size_t* dev_bytes);

/* dev_buf: device, 256-byte aligned, at least *dev_bytes from the query.  The
 * handle keeps dev_buf; the caller keeps it alive while the handle is used. */
uw_status uw_compress_commit(uw_blob* blob, const uint16_t* W_dev, void* scratch,
                             size_t scratch_bytes, void* dev_buf, size_t dev_bytes, void* stream);

/* Shape, palette, code, statistics and section table of a blob. */
uw_status uw_blob_info_get(const uw_blob* blob, uw_blob_info* info);

/* Device pointer and byte length of one section of a committed blob. */
uw_status uw_blob_section(const uw_blob* blob, int section, const void** dev_ptr, size_t* bytes);

/* Serialized size in bytes (header + format sections; the LUT is rebuilt on load). */
uw_status uw_blob_serialized_bytes(const uw_blob* blob, size_t* bytes);

/* Copies header and sections into host memory (synchronizes `stream`).  The
 * result is the "distribution bundle" form of §Llama 3.1 8B測試結果. */
uw_status uw_blob_serialize(const uw_blob* blob, void* host_dst, size_t cap, size_t* written,
                            void* stream);

/* Device image size needed to load a serialized blob (validates the header). */
uw_status uw_blob_device_bytes(const void* host_src, size_t n, size_t* dev_bytes);

/* Validates and loads a serialized blob into dev_buf (synchronizes `stream`).
 * Returns UW_ERR_CORRUPT if any size, offset, code or count is inconsistent. */
uw_status uw_blob_deserialize(const void* host_src, size_t n, void* dev_buf, size_t dev_bytes,
                              void* stream, uw_blob** out);

/* Frees the host handle only; device memory is the caller's. */
void uw_blob_free(uw_blob* blob);

/* ---------------------------------------------------------------- decode
 * HBM-to-HBM decoders of the Huffman form (§四種執行管道).  A stream the
 * decoder cannot parse sets UW_ERR_DEVICE in the device status word; output
 * is then unspecified, but no access leaves the blob's sections or the output. */

/* Full decode: W_out [N,K] BF16 bit patterns, bit-identical to the input of
 * compression.  W_out 16-byte aligned. */
uw_status uw_decode_full(const uw_blob* blob, uint16_t* W_out, void* stream);

/* Exponent-only decode: E_out[N*K] = exponent byte of every weight (verbatim
 * groups included).  E_out 16-byte aligned. */
uw_status uw_decode_exponent(const uw_blob* blob, uint8_t* E_out, void* stream);

/* Palette transcode: idx_out[N*K/2], byte-identical to the stored index
 * plane of the palette form.  idx_out 16-byte aligned. */
uw_status uw_transcode_palette(const uw_blob* blob, uint8_t* idx_out, void* stream);

/* ---------------------------------------------------------------- GEMM
 * Y[M,N] = X[M,K] . W^T with W given compressed (§重建矩陣乘法核心運作).
 * X: device BF16 [M,K], 16-byte aligned; Y: device [M,N] BF16 or float32.
 * M = 0 is a no-op.  Accumulation is float32 on the tensor cores, except
 * with UW_VARIANT_GEMV, or with UW_VARIANT_AUTO for M = 1 on a projection
 * with fewer than grid/2 tiles of 128 rows (grid: the GEMM CTA count, one
 * per SM by default) and sm_dec = 0: those run on the CUDA cores (a GEMV that
 * rebuilds the weights in registers).  The choice depends on the shape and
 * options only, so all pipelines and uw_dense_gemm take the same summation
 * order for a given M, N, K, variant, grid and split_k and agree bit for bit.
 * Every device-side wait is bounded: UW_TIMEOUT_MS (environment, read once,
 * default 2000, at least 10) milliseconds, after which the kernel raises
 * UW_ERR_TIMEOUT in the device status word and returns.  For tests of that
 * path, UW_DEBUG_SKIP_DECODER=1 (environment, read once) makes a
 * decoder-beside-GEMM call (sm_dec > 0) launch its GEMM without the decoder,
 * so the GEMM's waits for decoded bands run out.
 * Kernels are launched with programmatic dependent launch.  The direct-palette
 * pipeline requests its first weight tiles from the blob's device image
 * before waiting for the preceding kernel on the stream to finish, so that
 * image must not be written by device work that may still be running when
 * the call is enqueued (the library never writes a committed blob; ordinary
 * kernels and copies finish before a dependent kernel starts). */

/* Workspace bytes for uw_gemm with these options and M (UW_PIPE_AUTO: for the
 * plan's choice). */
uw_status uw_gemm_workspace(const uw_blob* blob, int64_t M, const uw_gemm_opts* opts, size_t* bytes);

/* UW_PIPE_AUTO lookup: copies into *out the options the plan gives for
 * (opts->projection, M) -- the entry of that projection with exactly M, else
 * the largest tuned M below it, else the smallest tuned M -- keeping out_f32,
 * workspace and stages from opts.  A concrete pipeline is copied unchanged.
 * UW_ERR_INVALID_ARG when the plan has no entry for the projection. */
uw_status uw_plan_resolve(const uw_gemm_opts* opts, int64_t M, uw_gemm_opts* out);

uw_status uw_gemm(const uint16_t* X, int64_t M, const uw_blob* blob, void* Y,
                  const uw_gemm_opts* opts, void* stream);

/* The uncompressed baseline: the same GEMM (tensor cores, or the GEMV where
 * uw_gemm would use it) on a plain BF16 W.  variant, grid and split_k as in
 * uw_gemm_opts. */
uw_status uw_dense_gemm_workspace(int64_t M, int64_t N, int64_t K, int variant, int grid, int split_k,
                                  size_t* bytes);

uw_status uw_dense_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N, int64_t K,
                        void* Y, int out_f32, int variant, int grid, int split_k, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- layer sequences
 * §跨層管道化: layers whose weights need a runtime Huffman decode ("hard")
 * alternate with layers kept in the pre-converted palette form ("easy"), so
 * that decompression never runs twice in a row and the decode of a hard
 * layer overlaps the matmul of the easy layer before it.  uw_gemm_sequence
 * runs a list of projections in order on `stream` (item i may read what item
 * i-1 wrote); every hard item's palette transcode runs on a library side
 * stream into one of two workspace buffers, as early as its buffer allows
 * (after the GEMM of the hard item two before it), and its GEMM waits for
 * it.  dec_ctas > 0: the transcodes run as that many small decoder CTAs that
 * fit beside the GEMM CTAs (which then leave room for one), so decode and
 * matmul share the SMs; 0: the standalone decoder.  The result of each item
 * equals uw_gemm of that item alone (transcode pipeline for hard items,
 * direct palette for easy ones, tensor cores) bit for bit.  Items on one
 * device that run beside each other in two calls at once must not overlap
 * (they share the side stream's events). */
typedef struct {
    const uw_blob* blob;
    const uint16_t* X;       /* device BF16 [M, K]                                       */
    void* Y;                 /* device [M, N], BF16 or float32 (out_f32)                 */
    int32_t hard;            /* 1: from the Huffman form (needs it); 0: from the palette form */
} uw_seq_item;

uw_status uw_sequence_workspace(const uw_seq_item* items, int n, int64_t M, size_t* bytes);

uw_status uw_gemm_sequence(const uw_seq_item* items, int n, int64_t M, int out_f32, int dec_ctas,
                           void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- gate + up, SwiGLU
 * §未來方向 names SwiGLU as the activation of the MLP: the gate and up
 * projections read the same X, and the down projection reads
 *   H[M,N] = silu(X . Wg^T) * (X . Wu^T),   silu(z) = z / (1 + e^-z).
 * uw_gemm_swiglu computes H in one launch from the palette forms of both
 * matrices: every tile of 128 rows carries the gate and the up rows, each
 * stage stages both matrices' tiles, TMEM holds two accumulators, and the
 * epilogue applies the SwiGLU in float32 before rounding H to BF16 (or
 * writing float32 with out_f32).  X is read once per tile for both products
 * and neither product goes to HBM.
 *   gate, up: committed blobs of the same shape [N, K] holding the palette
 *     form; X: device BF16 [M, K]; H: device [M, N].
 *   opts: pipeline UW_PIPE_DIRECT_PALETTE (others: UW_ERR_UNSUPPORTED),
 *     variant UW_VARIANT_AUTO or UW_VARIANT_TENSOR, sm_dec 0; grid, split_k,
 *     stages, out_f32 and the workspace as in uw_gemm.  Batch tiles are at
 *     most 128 rows (two accumulators share TMEM with the rebuilt tiles).
 * Above 128 batch rows the paired tile would need twice the rebuild work of
 * a 256-row single-matrix tile, so H is computed in three launches on the
 * same stream instead: the gate and the up projection, each with 256-row
 * tiles, into float32 blocks in the workspace, then an elementwise kernel
 * writing silu(G) * U.  The workspace size (uw_gemm_swiglu_workspace) covers
 * either form. */
uw_status uw_gemm_swiglu_workspace(const uw_blob* gate, const uw_blob* up, int64_t M, const uw_gemm_opts* opts,
                                   size_t* bytes);

uw_status uw_gemm_swiglu(const uint16_t* X, int64_t M, const uw_blob* gate, const uw_blob* up, void* H,
                         const uw_gemm_opts* opts, void* stream);

/* ---------------------------------------------------------------- allocation-free GEMM
 * An addition of this library; the pages have no counterpart.
 *
 * uw_gemm with the direct-palette pipeline for callers that cannot allocate
 * device memory at call time: engines that reserve all memory at start-up and
 * forbid allocation afterwards, code that must not risk the implicit device
 * synchronisation of cudaMalloc/cudaFree, plugins whose host framework owns
 * the allocator.  Its scratch (stream-K partial sums and arrival tags) is a
 * fixed 4 MiB array inside the library, present on every GPU that loads the
 * library until the process exits; no workspace argument, no allocation.
 *   X: device BF16 [M,K], 16-byte aligned; Y: device [M,N], BF16 or float32
 *   (out_f32), 16-byte aligned; the blob must hold the palette form.
 * Limits: returns UW_ERR_WORKSPACE, launching nothing, when the scratch this
 * call needs exceeds 4 MiB (on a 148-SM B200 that admits M <= 16, any N).  The array's contents carry over from call to call; they
 * need no clearing because every entry is tagged with its call.  All calls
 * share the one array, so calls that overlap on the GPU (other streams,
 * other threads) race: run them one at a time.  The first call on a device
 * looks the array's device address up (cudaGetSymbolAddress); make that first
 * call before any stream capture. */
uw_status uw_gemm_direct_palette_noalloc(const uint16_t* X, int64_t M, const uw_blob* blob, void* Y,
                                         int out_f32, void* stream);

/* ---------------------------------------------------------------- autotune
 * §自動調優機制: a measured coordinate descent.  For each batch size in Ms:
 * start every projection at the first feasible candidate, then sweep the
 * candidates of projection 0 with the others fixed, then 1, then 2, ..., and
 * repeat until a full round brings no improvement of more than 1%.  The cost
 * of a configuration is the device time (CUDA events) of the whole sequence
 * of projections, run `reps` times; pass r uses copy r % ncopies of every
 * projection, so with enough copies no weight is still in L2 from the pass
 * before.  Candidates: the four pipelines (those the blob's forms allow), the
 * matmul variants (batch 1: GEMV or tensor cores), an alternative grid (one
 * CTA per SM instead of the default rule) and, for the decoding pipelines,
 * decoder CTAs beside the GEMM (sm_dec = SMs/2, SMs, 2 SMs).  A candidate
 * whose call fails or whose kernels raise the device status (a bounded wait
 * that expired) counts as infeasible.
 *   blobs[c * nproj + i]: copy c of projection i (copies of one projection
 *     have the same shape); X[i], Y[i]: device buffers for the input (at
 *     least max(Ms) x K_i, BF16) and output (max(Ms) x N_i, BF16);
 *   workspace: at least the largest uw_gemm_workspace over the candidates
 *     (candidates that need more are skipped);
 *   plan_out: nproj * nM entries, written in (M, projection) order, each with
 *     the projection's own time (measured alone over the copies) and the
 *     whole sequence's time;
 *   plan_json_path: if not NULL, the plan is written there as JSON, with
 *     every measured trial ("trials": M, round, projection, candidate, time),
 *     and can be read back with uw_plan_load_json.
 * Synchronizes `stream`. */
uw_status uw_autotune(const uw_blob* const* blobs, int nproj, int ncopies, const int64_t* Ms, int nM,
                      const uint16_t* const* X, void* const* Y, void* workspace,
                      size_t workspace_bytes, int reps, uw_plan_entry* plan_out,
                      const char* plan_json_path, void* stream);

/* Reads the "plan" entries of a JSON file written by uw_autotune (the
 * per-model configuration file of §自動調優機制).  *n = entries found; at
 * most `cap` are stored.  UW_ERR_CORRUPT if the file holds no plan or an entry
 * lacks a field; UW_ERR_INVALID_ARG if it cannot be opened. */
uw_status uw_plan_load_json(const char* path, uw_plan_entry* entries, int cap, int* n);

#ifdef __cplusplus
}
#endif

#endif /* UNWEIGHT_H */
