/*
 * unweight.h - C ABI of libunweight: lossless BF16 weight compression fused
 * with the matmul that consumes the weights, for NVIDIA B200 (sm_100a).
 *
 * Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
 * sacrificing quality" (cited as *Unweight* with the section heading).
 *
 *   - "How model weights compress effectively": a BF16 weight is sign (1 bit),
 *     exponent (8 bits), mantissa (7 bits).
 *   - "Exponents are surprisingly predictable": sign and mantissa are kept
 *     verbatim; the exponent byte is Huffman coded; the 16 most frequent
 *     exponents form a palette; a 64-weight row holding any exponent outside
 *     the palette is stored verbatim.
 *   - "Four ways to use compressed weights": full decode to BF16 + plain GEMM;
 *     exponent-only decode; runtime palette transcode; palette transcoded once
 *     at load.  The last three feed a reconstructive matmul.
 *   - "How the reconstructive matmul works": compressed tiles are staged in
 *     shared memory, rebuilt to BF16 there and fed to the tensor cores; the
 *     rebuilt weights never reach main memory.
 *   - "Sharing the GPU between decode and compute": the decoder's ~16 KB
 *     lookup table, the decoder/GEMM SM split, the autotuner, easy/hard layers
 *     overlapped on side streams.
 *
 * Conventions (every call):
 *   - Weights W are [N, K] row-major BF16 bit patterns (torch Linear.weight);
 *     activations X are [M, K] row-major BF16; outputs Y are [M, N] row-major.
 *     K must be a positive multiple of 64.
 *   - "_dev" pointers are CUDA device pointers owned by the caller; "_host"
 *     pointers are host memory owned by the caller.  The library never frees a
 *     caller pointer and never keeps one after the call returns (except the
 *     workspace registered with uw_set_workspace, see there).
 *   - Device calls are asynchronous on the stream bound to the handle
 *     (uw_set_stream; default: the legacy default stream).  Argument errors are
 *     detected on the host before anything is launched.  Kernel-side errors
 *     (corrupt stream, bounded wait expired) set a status word in the handle,
 *     read by uw_last_device_status.  No call aborts, traps or throws.
 *   - Launch overlap: every kernel of the library is launched with programmatic
 *     stream serialization (CUDA programmatic dependent launch).  It may begin
 *     its set-up (barriers, tensor memory, decode tables, reads of the handle's
 *     own compressed arrays) while the kernel before it on the stream is still
 *     running, and waits for that kernel to complete (griddepcontrol.wait)
 *     before it reads or writes anything else: X, Y, workspaces, outputs.  So
 *     stream order holds for the caller's buffers exactly as with ordinary
 *     launches, also when the kernel before is the caller's own.
 *   - Thread safety: a handle may be used by one host thread at a time.
 */
#ifndef UNWEIGHT_H
#define UNWEIGHT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define UW_ABI_VERSION 1

#if defined(__GNUC__)
#define UW_API __attribute__((visibility("default")))
#else
#define UW_API
#endif

typedef enum uw_status {
  UW_OK = 0,
  UW_ERR_ARG = 1,          /* null pointer, bad enum, bad option value          */
  UW_ERR_SHAPE = 2,        /* N, K or M out of range, K not a multiple of 64    */
  UW_ERR_FORMAT = 3,       /* encoded data fails validation                     */
  UW_ERR_UNSUPPORTED = 4,  /* valid request this build cannot serve             */
  UW_ERR_OOM = 5,          /* device or host allocation failed                  */
  UW_ERR_CUDA = 6,         /* a CUDA runtime call failed                        */
  UW_ERR_DEVICE = 7,       /* a kernel reported corrupt input                   */
  UW_ERR_TIMEOUT = 8,      /* a kernel's bounded wait expired                   */
  UW_ERR_WORKSPACE = 9,    /* the pipeline needs a (larger) workspace           */
  UW_ERR_IO = 10           /* a file could not be opened, read or written       */
} uw_status;

/* Execution pipelines (*Unweight*, "Four ways to use compressed weights"). */
typedef enum uw_pipeline {
  UW_PIPE_AUTO = 0,            /* per-(M) choice from the loaded profile, else a default */
  UW_PIPE_FULL = 1,            /* Huffman decode to BF16 in HBM, then plain GEMM         */
  UW_PIPE_EXP = 2,             /* decode exponent bytes to HBM, reconstructive GEMM      */
  UW_PIPE_PALETTE_RT = 3,      /* transcode to 4-bit palette indices, reconstructive GEMM */
  UW_PIPE_PALETTE_DIRECT = 4,  /* palette indices prepared at load, reconstructive GEMM  */
  /* Beyond the four: the Huffman-direct product (*Unweight*, "How the
   * reconstructive matmul works": decoding inside the matmul moves about 30 %
   * fewer weight bytes than the palette form).  One kernel decodes the stream
   * and multiplies the rebuilt BF16 weights with X in warp-level MMAs (FP32
   * accumulation) as they decode; it reads the stream and the sign+mantissa
   * bytes (about 1.33 bytes per weight) and writes only Y.  M <= 8; K a
   * multiple of chunk_syms (UW_ERR_UNSUPPORTED otherwise).  Partial sums live
   * in the workspace (uw_workspace_bytes); no preprocessing pass.  Calls on
   * one handle must not overlap on the GPU (row counters in the handle).    */
  UW_PIPE_HUFFMAN_DIRECT = 5
} uw_pipeline;

/* Encoder options.  uw_default_encode_opts fills the defaults. */
typedef struct uw_encode_opts {
  int32_t max_code_len;    /* Huffman length cap, 1..12 (default 12: a 2^12-entry
                              4-byte decode table is 16 KB, "Sharing the GPU ...") */
  int32_t chunk_syms;      /* symbols per independently decodable chunk; a positive
                              multiple of 64 (default 256)                         */
  int32_t prepare_direct;  /* nonzero: at upload, transcode once into resident
                              palette indices so UW_PIPE_PALETTE_DIRECT works      */
  int32_t reserved;
} uw_encode_opts;

/*
 * Read-only view of an encoded matrix (host pointers).  Layout of each array:
 *   sm        [N*K]  u8  sign<<7 | mantissa, row-major
 *   code_len  [256]  u8  Huffman code length of each exponent value (0 = absent);
 *                        codes are canonical (RFC 1951 section 3.2.2)
 *   words     [n_words] u32  codes of E in row-major order, MSB first: stream bit
 *                        p is bit 31 - p%32 of words[p/32]; n_words % 4 == 0
 *   chunk_off [n_chunks+1] u32  start bit of each chunk of chunk_syms symbols;
 *                        chunk_off[n_chunks] = total bits
 *   palette   [16]   u8  the 16 most frequent exponents, ascending
 *   esc_bits  [(K/64) * NWp] u32, NWp = 4*ceil(N/128): bit n%32 of word
 *                        [kb*NWp + n/32] set when the 64-weight row (n, kb) is an
 *                        escape row (16 bytes per 128-row block; padding bits 0)
 *   esc_off   [n_esc_groups+1] u32  groups are (n/128, kb) in row-major order;
 *                        group g owns escape rows esc_off[g] .. esc_off[g+1]-1
 *   esc_exp   [n_esc_rows*64] u8  verbatim exponent bytes of each escape row
 */
typedef struct uw_format {
  int64_t N, K;
  int32_t max_code_len, chunk_syms;
  uint8_t code_len[256];
  uint8_t palette[16];
  int64_t n_words;       const uint32_t* words;
  int64_t n_chunks;      const uint32_t* chunk_off;
  const uint8_t* sm;
  int64_t n_esc_words;   const uint32_t* esc_bits;
  int64_t n_esc_groups;  const uint32_t* esc_off;
  int64_t n_esc_rows;    const uint8_t* esc_exp;
} uw_format;

typedef struct uw_stats_t {
  int64_t N, K;
  double bits_per_exponent;   /* Huffman stream bits / (N*K)                 */
  double entropy_bits;        /* empirical exponent entropy                  */
  double top16_coverage;      /* fraction of weights whose E is in the palette */
  int64_t n_rows, n_escape_rows;
  int32_t max_len_used, n_symbols;
  int64_t bytes_stream, bytes_offsets, bytes_sm, bytes_escape, bytes_palette_idx;
  int64_t bytes_huffman_bundle;   /* stream + offsets + S + code lengths          */
  int64_t bytes_palette_bundle;   /* indices + S + escape rows/bits/offsets       */
} uw_stats_t;

/* Explicit GEMM variant (what the autotuner chooses; 0 = library default). */
typedef struct uw_gemm_config {
  int32_t pipeline;      /* uw_pipeline, not AUTO                                  */
  int32_t tile_n;        /* tokens per MMA tile: 16..256, multiple of 16 (0=auto)  */
  int32_t stages;        /* weight load-ring depth, 2..16, even unless halves=2
                            (0 = auto; X tiles have their own, automatic ring)      */
  int32_t gemm_ctas;     /* persistent GEMM CTAs (0 = one per SM); pipeline 5: the
                            SMs (one CTA each) of its single kernel                 */
  int32_t decode_ctas;   /* SMs (one CTA each) of the preprocessing kernel (0 = all) */
  int32_t halves;        /* W rows per GEMM unit / 128: 1, or 2 (the wide shape: X
                            is read once per 256 rows); 0 = 1                       */
  int32_t pair;          /* 1: the BF16 GEMM (pipeline 1) on CTA pairs: one two-SM
                            MMA of 256 W rows x 256 tokens per step over an SM pair,
                            each CTA loading its 128 rows and half of the tokens
                            (256-token tiles; one half per unit); 0: one CTA per
                            tile.  Other pipelines: UW_ERR_UNSUPPORTED              */
  int32_t gemv;          /* 1: the matrix-vector kernel on the CUDA cores, M <= 2 only
                            (each weight rebuilt in registers and multiplied in FP32,
                            no tensor cores; UW_ERR_UNSUPPORTED above M = 2); 0: the
                            tensor-core GEMM.  The autotuner tries 1 at M <= 2.
                            Pipeline 5 (always on the CUDA cores): must be 0.
                            Pipeline 5 ignores tile_n, stages, halves, decode_ctas */
} uw_gemm_config;

typedef struct uw_host_s* uw_host_t;       /* host-side encoded matrix         */
typedef struct uw_handle_s* uw_handle_t;   /* device-resident encoded matrix   */

/* Human-readable name of a status code (static string, never NULL). */
UW_API const char* uw_status_str(uw_status s);
UW_API int uw_abi_version(void);
UW_API void uw_default_encode_opts(uw_encode_opts* opts);

/* ---- host side (no GPU needed) ------------------------------------------- */

/* Compress W (host, [N, K] BF16 bits) on the host.  Steps ("Exponents are
 * surprisingly predictable"): exponent histogram, palette, escape rows,
 * optimal length-limited code lengths (package-merge, cap max_code_len),
 * canonical codes, chunked bitstream with bit offsets, S stream.
 * Errors: UW_ERR_ARG (null), UW_ERR_SHAPE (N<1, K<64, K%64), UW_ERR_UNSUPPORTED
 * (stream above 2^32 - 128 bits), UW_ERR_OOM.  *out is owned by the caller:
 * uw_host_free. */
UW_API uw_status uw_encode_host(const uint16_t* w_host, int64_t N, int64_t K,
                         const uw_encode_opts* opts, uw_host_t* out);
/* Fill *view with pointers into h (valid until uw_host_free(h)). */
UW_API uw_status uw_host_view(uw_host_t h, uw_format* view);
UW_API void uw_host_free(uw_host_t h);
/* Structural validation of an encoded matrix: shapes, Kraft inequality, length
 * cap, monotone chunk offsets within the stream, per-chunk bit counts between
 * min and max code length, distinct palette, escape bitmap consistent with
 * the group offsets.  UW_OK or UW_ERR_FORMAT / UW_ERR_SHAPE / UW_ERR_ARG, or
 * UW_ERR_UNSUPPORTED for a stream longer than 2^27 - 4 words. */
UW_API uw_status uw_validate_format(const uw_format* f);
/* Statistics of a host-side encoding (no GPU). */
UW_API uw_status uw_host_stats(uw_host_t h, uw_stats_t* out);

/* Distribution bundle (*Unweight*, the untitled passage on format and execution:
 * the Huffman package is what is shipped, and at load it is transcoded to the
 * form inference runs on).  uw_host_save writes h to `path`: a 16-byte-aligned
 * little-endian file holding the header (shape, code lengths, palette, exponent
 * histogram, array sizes), the arrays of uw_format in their order, then a 64-bit
 * FNV-1a checksum of all preceding bytes and an end tag.  uw_host_load reads such
 * a file into a new host encoding (owned by the caller: uw_host_free) after
 * checking the tag, the checksum, the header, uw_validate_format, and that the
 * histogram counts the N*K exponents with a code for every counted one.  Errors:
 * UW_ERR_ARG (null), UW_ERR_IO (open, read or write failed), UW_ERR_FORMAT
 * (truncated, corrupted or not a bundle), UW_ERR_SHAPE, UW_ERR_OOM. */
UW_API uw_status uw_host_save(uw_host_t h, const char* path);
UW_API uw_status uw_host_load(const char* path, uw_host_t* out);

/* ---- device side ---------------------------------------------------------- */

/* Validate f, copy it to the current CUDA device on `stream` (a cudaStream_t,
 * may be NULL), build the decode tables, and if opts->prepare_direct run the
 * load-time palette transcode.  The host data is not retained.  *out is
 * owned by the caller: uw_free.  Errors: as uw_validate_format, UW_ERR_OOM,
 * UW_ERR_CUDA. */
UW_API uw_status uw_upload(const uw_format* f, const uw_encode_opts* opts, void* stream,
                    uw_handle_t* out);
/* uw_host_load + uw_upload: a bundle straight to the device (with the load-time
 * palette transcode when opts->prepare_direct; opts may be NULL for the
 * defaults).  Errors: as uw_host_load and uw_upload. */
UW_API uw_status uw_load(const char* path, const uw_encode_opts* opts, void* stream,
                         uw_handle_t* out);
/* uw_encode_host + uw_upload (the load-time entry point). */
UW_API uw_status uw_encode(const uint16_t* w_host, int64_t N, int64_t K,
                    const uw_encode_opts* opts, void* stream, uw_handle_t* out);
UW_API uw_status uw_free(uw_handle_t h);
UW_API uw_status uw_set_stream(uw_handle_t h, void* stream);
UW_API uw_status uw_stats(uw_handle_t h, uw_stats_t* out);

/* Workspace: pipelines FULL, EXP and PALETTE_RT write their preprocessed
 * weights (2*N*K, N*K, N*K/2 bytes) and the GEMM its split-K partial sums to a
 * device workspace; HUFFMAN_DIRECT keeps its per-row partial sums there
 * (32 bytes per chunk of the stream).  uw_workspace_bytes gives a size that
 * serves (pipeline, M) with any variant (token tile up to 256, up to one CTA
 * per SM), or UW_ERR_UNSUPPORTED where the pipeline does not serve M;
 * uw_set_workspace registers caller-owned device memory (kept by pointer until
 * replaced or the handle is freed; ptr NULL unregisters); uw_alloc_workspace
 * makes the handle allocate and own one of `bytes` bytes.  Calls that need
 * more workspace than registered return UW_ERR_WORKSPACE and launch nothing.
 * A tile whose K range is split between CTAs is summed inside the GEMM
 * kernel, through the workspace and a small hand-off block the handle owns;
 * so a handle's calls must be ordered (one stream, or synchronised streams):
 * two of its GEMMs running at the same time race. */
UW_API uw_status uw_workspace_bytes(uw_handle_t h, int32_t pipeline, int64_t M, size_t* bytes);
UW_API uw_status uw_set_workspace(uw_handle_t h, void* ws_dev, size_t bytes);
UW_API uw_status uw_alloc_workspace(uw_handle_t h, size_t bytes);

/* Full Huffman decode ("Four ways...", pipeline 1 preprocessing): writes the
 * N*K BF16 weights to w_dev (caller-owned, 16-byte aligned).  Bit-exact. */
UW_API uw_status uw_decode_full(uw_handle_t h, uint16_t* w_dev);
/* Row gather on compressed weights: the BF16 rows rows_dev[0 .. n_rows-1] of
 * W (an embedding lookup: token ids into a [vocab, dim] table) decoded into
 * w_dev, [n_rows, K] row-major, row i of the output = row rows_dev[i] of W.
 * Only the requested rows' chunks are decoded (the same table-driven decoder
 * as uw_decode_full).  "Exponents are surprisingly predictable" and the
 * closing remarks of *Unweight*: the format is not specific to MLP weights.
 * rows_dev: device int64 array, 8-byte aligned; ids may repeat; an id outside
 * [0, N) leaves its output row unspecified and makes uw_last_device_status
 * report UW_ERR_DEVICE.  w_dev 16-byte aligned.  Needs K to be a multiple of
 * the encoding's chunk_syms (UW_ERR_UNSUPPORTED otherwise).  n_rows == 0
 * returns UW_OK and launches nothing. */
UW_API uw_status uw_decode_rows(uw_handle_t h, const int64_t* rows_dev, int64_t n_rows,
                                uint16_t* w_dev);
/* Exponent-only decode (pipeline 2 preprocessing): N*K exponent bytes to e_dev
 * (16-byte aligned), row-major. */
UW_API uw_status uw_decode_exp(uw_handle_t h, uint8_t* e_dev);
/* Palette transcode (pipeline 3 preprocessing; also the load-time step of
 * pipeline 4): N*K/2 bytes of packed 4-bit indices to idx_dev (16-byte
 * aligned).  Index i of element (n, k) is the rank of its exponent in the
 * ascending palette.  Each group of 8 consecutive elements of a row is one
 * little-endian 32-bit word: element 2t at bits 4t..4t+3, element 2t+1 at bits
 * 16+4t..16+4t+3 (t = 0..3), so each 16-bit half holds one index of every
 * BF16 pair in the pair's own lane.  All indices of an escape row are 0. */
UW_API uw_status uw_transcode_palette(uw_handle_t h, uint8_t* idx_dev);

/* Y[M, N] = X[M, K] W^T with BF16 inputs, FP32 accumulation, BF16 output
 * (round to nearest even).  pipeline AUTO takes the profile's choice for M.
 * M == 0 returns UW_OK and launches nothing.  X and Y are device pointers,
 * 16-byte aligned, row-major, not overlapping. */
UW_API uw_status uw_gemm(uw_handle_t h, const uint16_t* X_dev, uint16_t* Y_dev, int64_t M,
                  uw_pipeline pipeline);
/* As uw_gemm with FP32 output (no final rounding). */
UW_API uw_status uw_gemm_f32(uw_handle_t h, const uint16_t* X_dev, float* Y_dev, int64_t M,
                      uw_pipeline pipeline);
/* As uw_gemm / uw_gemm_f32 with an explicit variant; out_f32 selects the
 * output type of Y_dev (float* when nonzero, uint16_t* BF16 otherwise). */
UW_API uw_status uw_gemm_ex(uw_handle_t h, const uint16_t* X_dev, void* Y_dev, int64_t M,
                     const uw_gemm_config* cfg, int32_t out_f32);

/* Allocation-free matmul, pipeline 4 only (the paper has no counterpart to
 * this call; it exists for callers that cannot allocate).  Some callers cannot
 * allocate device memory while they run a matmul: their allocator is locked or
 * already committed to a fixed memory plan, or they run where a cudaMalloc
 * would stall or fail.  uw_gemm needs a registered workspace for split-K
 * partial sums; this call keeps them in a fixed array compiled into the
 * library instead, so it allocates nothing (no cudaMalloc, no workspace).
 *   - Computes Y[M, N] = X W^T like uw_gemm(..., UW_PIPE_PALETTE_DIRECT);
 *     Y is float* when out_f32 is nonzero, else BF16.  Needs a handle
 *     uploaded with prepare_direct (UW_ERR_UNSUPPORTED otherwise).
 *   - Limit: M <= 64 (UW_ERR_SHAPE above that).  The array is 5 MiB and is
 *     held on every GPU where the library's device code is loaded, until the
 *     process exits.
 *   - When the array is allocated: the CUDA driver allocates it when it loads
 *     the library module that holds it.  uw_upload / uw_encode / uw_load with
 *     prepare_direct load that module and look up the array's device address
 *     on the handle's device, so the 5 MiB are taken at load time, not by this
 *     call.  (Only if no such upload happened on the device does the first
 *     call do the lookup itself; make that first call before any stream
 *     capture.)
 *   - The handle's device must be current (UW_ERR_ARG otherwise).
 *   - All calls on one GPU share the one array: calls whose kernels overlap
 *     on that GPU (for example on two streams) race and give wrong results.
 *     Nothing in it needs to start at zero, and its contents after a call
 *     are meaningless. */
UW_API uw_status uw_gemm_palette_noalloc(uw_handle_t h, const uint16_t* X_dev, void* Y_dev,
                                         int64_t M, int32_t out_f32);

/* Autotuner ("Sharing the GPU between decode and compute", last paragraphs):
 * for every M in Ms, coordinate descent over the handles (projections): each
 * handle in turn tries every candidate variant (pipeline, token tile, ring
 * depth) while the others keep theirs, scored by the device time (CUDA
 * events on the first handle's stream) of all handles' matmuls in order;
 * sweeps repeat until no change gains 1 %.  The winners are stored in the
 * handles (uw_gemm with UW_PIPE_AUTO uses them) and, when profile_out_json is
 * not NULL, written as JSON.  Candidates that need more workspace than a
 * handle has registered are skipped (UW_ERR_WORKSPACE when none fits).  The
 * tuner allocates its own X/Y buffers.  The decoder/GEMM SM split is tuned
 * for the overlapped stack by uw_mlp_tune_split. */
UW_API uw_status uw_autotune(uw_handle_t* hs, int32_t n_handles, const int64_t* Ms, int32_t n_M,
                      const char* profile_out_json);
/* Load a profile written by uw_autotune into the handles (matched by order and
 * shape).  UW_ERR_FORMAT on a malformed file or a shape mismatch. */
UW_API uw_status uw_load_profile(uw_handle_t* hs, int32_t n_handles, const char* profile_json);
/* The variant uw_gemm(..., UW_PIPE_AUTO) would use for M. */
UW_API uw_status uw_get_choice(uw_handle_t h, int64_t M, uw_gemm_config* cfg);

/* Kernel tracing.  While enabled, every kernel the handle launches is
 * bracketed by two CUDA events recorded on the handle's stream (no extra
 * synchronisation); the times are meaningful for calls that launch on that
 * stream (uw_gemm*, the decode calls), not for the MLP calls, which launch on
 * the streams they are given.  uw_trace_read synchronises the stream and returns, in
 * launch order, each recorded launch's kind (uw_kernel_kind) and device time
 * in milliseconds, then clears the record.  At most 16384 launches are kept;
 * *count gets the number recorded, of which min(count, capacity) are copied. */
typedef enum uw_kernel_kind {
  UW_KERNEL_DECODE_FULL = 0, UW_KERNEL_DECODE_EXP = 1, UW_KERNEL_TRANSCODE = 2,
  UW_KERNEL_GEMM_BF16 = 3, UW_KERNEL_GEMM_EXP = 4, UW_KERNEL_GEMM_PALETTE = 5,
  UW_KERNEL_SPLITK_FIXUP = 6,  /* reserved: split tiles are summed inside the GEMM */
  UW_KERNEL_GEMV_BF16 = 7, UW_KERNEL_GEMV_EXP = 8, UW_KERNEL_GEMV_PALETTE = 9,
  UW_KERNEL_DECODE_DOT = 10  /* the Huffman-direct product (UW_PIPE_HUFFMAN_DIRECT) */
} uw_kernel_kind;
UW_API uw_status uw_trace_enable(uw_handle_t h, int32_t enable);
UW_API uw_status uw_trace_read(uw_handle_t h, int32_t* kinds, float* ms, int32_t capacity,
                               int32_t* count);

/* ---- MLP stack ("Sharing the GPU between decode and compute") ------------ */

/* One SwiGLU block: gate and up are [F, D] weights, down is [D, F]. */
typedef struct uw_mlp_layer {
  uw_handle_t gate, up, down;
} uw_mlp_layer;

typedef struct uw_mlp_opts {
  int32_t overlap;      /* nonzero: projections whose pipeline needs preprocessing
                           ("hard": 1-3) are preprocessed on side_stream one hard
                           projection ahead, into two alternating workspace slots,
                           while the main stream runs the GEMMs                     */
  int32_t decode_ctas;  /* SM split, decoder share: SMs (one CTA each) of each
                           side-stream preprocessing kernel (0 = all of them)        */
  int32_t gemm_ctas;    /* SM split, GEMM share: CTAs of each GEMM while the stack
                           runs (0 = one per SM); a profile's own value wins         */
  int32_t reserved;
} uw_mlp_opts;

/* h[i] = SiLU(g[i]) * u[i] for n BF16 values (SiLU and product in FP32, result
 * rounded to nearest even); device pointers, 16-byte aligned, on `stream`. */
UW_API uw_status uw_swiglu(const uint16_t* g_dev, const uint16_t* u_dev, uint16_t* h_dev,
                           int64_t n, void* stream);
/* Workspace uw_mlp_forward needs for these layers, M and options. */
UW_API uw_status uw_mlp_workspace_bytes(const uw_mlp_layer* layers, int32_t n_layers, int64_t M,
                                        const uw_mlp_opts* opts, size_t* bytes);
/* x_0 = X [M, D]; x_{l+1} = (SiLU(x_l Wg^T) * (x_l Wu^T)) Wd^T; Y = x_L [M, D].
 * Each projection uses the variant its handle's profile picks for M (see
 * uw_autotune / uw_load_profile; default otherwise).  X, Y device pointers
 * (16-byte aligned, may alias); ws_dev caller-owned, 256-byte aligned, at least
 * uw_mlp_workspace_bytes; the handles' own workspaces are not used.  Work is
 * enqueued on `stream` (and side_stream when overlapping; the call orders it
 * after all earlier work on `stream`).  Errors as uw_gemm, UW_ERR_SHAPE when
 * the layers' shapes do not chain. */
UW_API uw_status uw_mlp_forward(const uw_mlp_layer* layers, int32_t n_layers, const uint16_t* X_dev,
                                uint16_t* Y_dev, int64_t M, void* ws_dev, size_t ws_bytes,
                                void* stream, void* side_stream, const uw_mlp_opts* opts);
/* uw_mlp_forward that also records every layer's intermediate activations,
 * for checking a compressed stack layer by layer against a reference.  act_dev
 * (caller-owned, 16-byte aligned) receives, per layer l, at element offset
 * l * M * (3F + D): g = x_l Wg^T [M, F], u = x_l Wu^T [M, F],
 * h = SiLU(g) * u [M, F], x_{l+1} = h Wd^T [M, D] (BF16, row-major; F and D
 * from the first layer's gate: [F, D]).  The copies are device-to-device on
 * `stream`, right after each value is produced; the arithmetic, the variants
 * and the overlap are those of uw_mlp_forward.  Errors as uw_mlp_forward, and
 * UW_ERR_ARG for a null or misaligned act_dev. */
UW_API uw_status uw_mlp_forward_record(const uw_mlp_layer* layers, int32_t n_layers,
                                       const uint16_t* X_dev, uint16_t* Y_dev, int64_t M,
                                       void* ws_dev, size_t ws_bytes, void* stream,
                                       void* side_stream, const uw_mlp_opts* opts,
                                       uint16_t* act_dev);
/* Decoder/GEMM SM split for the overlapped stack: time uw_mlp_forward (overlap
 * on) for a few (decode_ctas, gemm_ctas) pairs and no split, return the
 * fastest in *best.  Synchronises `stream`. */
UW_API uw_status uw_mlp_tune_split(const uw_mlp_layer* layers, int32_t n_layers,
                                   const uint16_t* X_dev, uint16_t* Y_dev, int64_t M, void* ws_dev,
                                   size_t ws_bytes, void* stream, void* side_stream,
                                   uw_mlp_opts* best);

/* Synchronise the handle's stream, then return and clear the device status
 * word: UW_OK, UW_ERR_DEVICE (a chunk decoded to the wrong bit count or hit an
 * invalid code) or UW_ERR_TIMEOUT (a bounded wait in a kernel expired). */
UW_API uw_status uw_last_device_status(uw_handle_t h);

#ifdef __cplusplus
}
#endif
#endif /* UNWEIGHT_H */
