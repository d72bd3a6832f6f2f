/*
 * mxattn.h -- C ABI of libmxattn.so: MXAttention's MXFP4 forward attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("MXAttention: Data-Free Optimal Scaling and Pre-Normalization
 * Quantization for MXFP4 Attention", as described on its Pith review page and
 * in the 10100.com article) computes, per attention head:
 *   1. a fixed orthonormal Hadamard rotation of every Q and K row (Fig. 1;
 *      axioms ledger, Sec. 4.3);
 *   2. MXFP4 quantization of Q, K and V: groups of 32 values share one E8M0
 *      power-of-two scale, each value becomes an E2M1 code (grid 0, +-0.5,
 *      +-1, +-1.5, +-2, +-3, +-4, +-6; round to nearest, ties to even,
 *      saturating at 6).  The scale exponent is the Universal Optimal
 *      Scaling ceiling rule with boundary Qmax = 7.25 (Fig. 3: the block
 *      maximum maps to (3.625, 7.25]); Qmax = 6 and the OCP floor rule are
 *      ablation options.  Q/K groups run along the head dimension, V groups
 *      along the key axis;
 *   3. a FlashAttention-2 style online softmax with Pre-Normalization
 *      Quantization (Fig. 4): every unnormalized exponential tile
 *      P~ = exp(S - m_running) is quantized to MXFP4 once and that same
 *      quantized tile feeds both the row sum l and the P~ V update.
 *
 * Conventions
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library allocates no memory, never synchronizes (except
 *    mxattn_get_device_error), and enqueues all work on `stream`, a
 *    cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Arguments are validated before anything is enqueued; an invalid call
 *    returns an error status and enqueues nothing.
 *  - q, k, v, out are contiguous [B, H, N, d] ("BHND") in opts->dtype; out
 *    has the input dtype.  Self-attention, N_q = N_k = N, without masking
 *    unless opts->causal; mxattn_forward_cross takes N_q != N_k and
 *    mxattn_forward_varlen a token-major packed batch (see there).
 *  - Codes are packed two per byte, element 2i in the LOW nibble, element
 *    2i+1 in the high nibble; bit 3 of a code is the sign (a negative value
 *    that rounds to zero keeps its sign: code 0x8).  Scales are E8M0 bytes
 *    (2^(byte-127)); the byte 0xFF is never written; an all-zero group gets
 *    byte 0x00 and zero codes.
 *
 * Packed attention-operand layouts (what mxattn_hadamard_quant_qk and
 * mxattn_quant_v write, what mxattn_attention_mxfp4 reads).  They are the
 * shared-memory images the tcgen05 block-scaled MMA consumes, so each tile is
 * moved with one bulk copy:
 *
 *  QK codes   [B*H][T128][128][d/2] bytes, T128 = ceil(N/128).  Tile t holds
 *             tokens 128t .. 128t+127 (rows past N are zero).  Row r of a
 *             tile is stored at byte r*(d/2); its 16-byte chunk c (= MX group
 *             c, elements 32c..32c+31) is stored at chunk position c ^ s(r):
 *               d = 128:  s(r) = (r >> 1) & 3     (64-byte swizzle)
 *               d =  64:  s(r) = (r >> 2) & 1     (32-byte swizzle)
 *  QK scales  [B*H][T128][512] bytes, one 512-byte scale atom per 128-row
 *             tile: the scale of token r (0..127 within the tile), group g
 *             (0..3) sits at byte (r % 32)*16 + (r / 32)*4 + g.  Groups
 *             g >= d/32 are zero.
 *  V codes    [B*H][T64][d][32] bytes, T64 = ceil(N/64): V is transposed so
 *             that each channel is a row of 64 keys (32 bytes).  Row c of
 *             tile j holds keys 64j .. 64j+63 of channel c; its 16-byte chunk
 *             h (keys 64j+32h .. +31, one MX group) sits at chunk position
 *             h ^ ((c >> 2) & 1).  Keys past N are zero.
 *  V scales   [B*H][T128][512] bytes: the atom of keys 128t .. 128t+127 holds
 *             the scale of channel c, key group g (0..3) at byte
 *             (c % 32)*16 + (c / 32)*4 + g.  Channels >= d are zero.
 *
 * NVFP4 comparison format (opts->format = MXATTN_FMT_NVFP4): the same codes,
 * in blocks of 16 elements whose scales are E4M3 bytes (FP8: bias 7, 3
 * mantissa bits, subnormals, largest 448; scale = E4M3(fl32(amax / 6)), codes
 * of fl32(x / scale), a zero scale gives zero codes).  The scale atoms hold
 * 4 blocks (64 elements) per row:
 *  QK scales  [B*H][T128][d/64][512]: atom a covers dims 64a .. 64a+63, block
 *             b (0..3) of token r at byte (r % 32)*16 + (r / 32)*4 + b.
 *  V scales   [B*H][T64][512]: one atom per 64-key tile, key block b (0..3)
 *             of channel c at byte (c % 32)*16 + (c / 32)*4 + b.
 * The pages compare MXAttention with NVFP4-based baselines without defining
 * NVFP4; this is the public format, built for that comparison (full attention,
 * no dump, no causal or varlen).  The exponential tile P~ <= 1 is scaled by
 * 448*6 before its blocks take their scales (the block holding the running
 * max gets scale 448); the factor cancels in O = O~/l.
 *
 * Workspace (mxattn_forward, mxattn_attention_mxfp4): opts->workspace is a
 * device buffer of at least mxattn_workspace_bytes() bytes, 256-byte aligned.
 * Its first 256 bytes are a status block that the kernels set when a bounded
 * device-side wait expires; zero it once with mxattn_workspace_init before
 * first use.  mxattn_forward keeps the packed Q/K/V operands after it.
 */
#ifndef MXATTN_H_
#define MXATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MXATTN_ABI_VERSION 1

#if defined(__GNUC__)
#define MXATTN_API __attribute__((visibility("default")))
#else
#define MXATTN_API
#endif

typedef enum mxattn_status {
  MXATTN_OK = 0,
  MXATTN_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad option value        */
  MXATTN_ERR_UNSUPPORTED = 2, /* valid but not implemented (d, key_tile, dtype)   */
  MXATTN_ERR_WORKSPACE = 3,   /* workspace missing, too small or misaligned       */
  MXATTN_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed              */
  MXATTN_ERR_TIMEOUT = 5      /* a bounded device-side wait expired (see below)   */
} mxattn_status;

typedef enum mxattn_scale_rule {
  MXATTN_SCALE_UOS = 0,        /* ceiling rule, boundary 29/4: max -> (3.625, 7.25] */
  MXATTN_SCALE_QMAX6 = 1,      /* ceiling rule, boundary 6:    max -> (3, 6]        */
  MXATTN_SCALE_OCP = 2,        /* OCP floor rule e = floor(log2 amax) - 2: [4, 8)  */
  MXATTN_SCALE_CEIL_CUSTOM = 3 /* ceiling rule, boundary opts.qmax in [4, 8]       */
} mxattn_scale_rule;

typedef enum mxattn_dtype { MXATTN_BF16 = 0, MXATTN_FP32 = 1 } mxattn_dtype;

typedef enum mxattn_format {
  MXATTN_FMT_MXFP4 = 0,  /* 32-element groups, E8M0 scale chosen by opts.scale_rule */
  MXATTN_FMT_NVFP4 = 1   /* 16-element blocks, E4M3 scale (comparison format)       */
} mxattn_format;

typedef struct mxattn_opts {
  int scale_rule;          /* mxattn_scale_rule, used for Q, K, V and the P~ tiles      */
  float qmax;              /* boundary for MXATTN_SCALE_CEIL_CUSTOM                      */
  int pnq;                 /* 1: l from the quantized tile (PNQ); 0: direct placement   */
  int rotate;              /* 1: Hadamard-rotate Q and K before quantizing               */
  int dtype;               /* mxattn_dtype of q, k, v, out                               */
  int key_tile;            /* keys per online-softmax step: 128 (the default, the       */
                           /* faster kernel) or 64; NVFP4 runs only with 64 (128 with   */
                           /* NVFP4 returns MXATTN_ERR_UNSUPPORTED).  The lazy running   */
                           /* max moves at tile boundaries, so results depend on it.     */
  float rescale_tau;       /* the running max moves only when it grows by more than    */
                           /* tau (log2 units); 0 = eager FlashAttention-2 update       */
  void* workspace;         /* device buffer, see mxattn_workspace_bytes                  */
  size_t workspace_bytes;  /* its size in bytes                                          */
  long long wait_budget_cycles; /* SM clock cycles a pipeline wait inside the attention     */
                           /* kernel may last before the kernel gives up and records     */
                           /* MXATTN_ERR_TIMEOUT; 0 = default (2e9, about one second).  */
                           /* A test sets it tiny to exercise the expiry path (a wait    */
                           /* is checked against it only after a first hardware try_wait */
                           /* returned without the phase); draining in-flight copies and */
                           /* MMAs always gets the default budget.                       */
  int causal;              /* 1: causal self-attention, query row i sees keys 0..i (an   */
                           /* autoregressive mask; the pages' video models attend both   */
                           /* ways and fix none); key tiles past a query tile's diagonal */
                           /* are skipped.  Self-attention entry points only (varlen:    */
                           /* within each sequence); cross-attention returns             */
                           /* MXATTN_ERR_UNSUPPORTED, as does NVFP4.  0 = full attention. */
  int format;              /* mxattn_format: MXFP4 (the method) or NVFP4 (comparison)     */
} mxattn_opts;

/* Fill *opts with the defaults: UOS, qmax 7.25, pnq 1, rotate 1, bf16,
 * key_tile 128, rescale_tau 8, no workspace, default wait budget, MXFP4,
 * causal 0.  (NVFP4 callers set key_tile = 64.) */
MXATTN_API void mxattn_opts_default(mxattn_opts* opts);

/* Bytes of workspace mxattn_forward needs for this problem (status block plus
 * packed Q, K, V operands); 0 for invalid sizes. */
MXATTN_API size_t mxattn_workspace_bytes(int B, int H, int N, int d, const mxattn_opts* opts);

/* Sizes of the packed attention operands described above (0 for invalid sizes),
 * MXFP4; NVFP4 needs d/64 times the QK scale bytes and ceil(N/64)*512 per head
 * for the V scales (mxattn_workspace_bytes takes the format from opts). */
MXATTN_API size_t mxattn_qk_codes_bytes(int B, int H, int N, int d);
MXATTN_API size_t mxattn_qk_scales_bytes(int B, int H, int N, int d);
MXATTN_API size_t mxattn_v_codes_bytes(int B, int H, int N, int d);
MXATTN_API size_t mxattn_v_scales_bytes(int B, int H, int N, int d);

/* The six sizes for the format in opts (MXFP4 or NVFP4), in the order q codes,
 * q scales, k codes, k scales, v codes, v scales, written to sizes[0..5].
 * Returns MXATTN_ERR_INVALID_ARG (sizes untouched) for invalid sizes or opts. */
MXATTN_API mxattn_status mxattn_operand_bytes(int B, int H, int N, int d, const mxattn_opts* opts,
                                              size_t* sizes);

/* Zero the workspace status block (enqueued on stream). */
MXATTN_API mxattn_status mxattn_workspace_init(const mxattn_opts* opts, void* stream);

/*
 * Generic MXFP4 quantization of a row-major [rows][cols] matrix x
 * (opts->dtype), with the scale rule of opts (10100.com article: 32-element
 * groups sharing one E8M0 scale; Fig. 3 of the paper for the rules).
 *  group_axis 0: groups of 32 consecutive columns of each row;
 *                codes [rows][ceil(cols/32)*16], scales [rows][ceil(cols/32)].
 *  group_axis 1: groups of 32 consecutive rows of each column, written
 *                transposed: codes [cols][ceil(rows/32)*16],
 *                scales [cols][ceil(rows/32)].
 * Partial tail groups are zero-padded.  No rotation is applied.
 * opts->format = MXATTN_FMT_NVFP4: blocks of 16 with E4M3 scale bytes
 * (codes [outer][ceil(inner/16)*8], scales [outer][ceil(inner/16)]).
 */
MXATTN_API mxattn_status mxattn_quantize_mxfp4(const void* x, int64_t rows, int64_t cols, int group_axis,
                                    const mxattn_opts* opts, uint8_t* codes, uint8_t* scales,
                                    void* stream);

/*
 * Step 1+2 for Q and K: Hadamard rotation (if opts->rotate) and MXFP4
 * quantization along d, written in the packed QK operand layout.
 * The rotation is y = x H_d / sqrt(d) for the natural-order Sylvester
 * Hadamard matrix, computed in fp32 as log2(d) butterfly stages
 * h = 1, 2, ..., d/2 ((a, b) -> (a + b, a - b)) followed by one multiply by
 * fl32(1/sqrt(d)); the scale rule reads these fp32 values.
 * d in {64, 128}.  Buffers: mxattn_qk_codes_bytes / mxattn_qk_scales_bytes.
 */
MXATTN_API mxattn_status mxattn_hadamard_quant_qk(const void* q, const void* k, int B, int H, int N, int d,
                                       const mxattn_opts* opts, uint8_t* q_codes,
                                       uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales,
                                       void* stream);

/*
 * Step 2 for V: MXFP4 quantization in groups of 32 consecutive keys per
 * channel (no rotation), written in the packed V operand layout.
 */
MXATTN_API mxattn_status mxattn_quant_v(const void* v, int B, int H, int N, int d, const mxattn_opts* opts,
                             uint8_t* v_codes, uint8_t* v_scales, void* stream);

/*
 * Step 3 alone on packed operands: S = Q^ K^T (block-scaled FP4 tensor-core
 * MMA, fp32 accumulation) times softmax_scale, online softmax over key tiles
 * of opts->key_tile keys, each exponential tile quantized to MXFP4 in groups
 * of 32 keys with the scale rule of opts, l updated from the quantized tile
 * (PNQ) or from the unquantized one (pnq = 0), O~ += P^ V^, O = O~ / l in
 * opts->dtype.  Requires opts->workspace (status block, >= 256 bytes).
 */
MXATTN_API mxattn_status mxattn_attention_mxfp4(const uint8_t* q_codes, const uint8_t* q_scales,
                                     const uint8_t* k_codes, const uint8_t* k_scales,
                                     const uint8_t* v_codes, const uint8_t* v_scales, int B, int H,
                                     int N, int d, float softmax_scale, const mxattn_opts* opts,
                                     void* out, void* stream);

/*
 * Scale-rule diagnostic: per-block Qmax sweep (the per-block MSE-optimal
 * boundary study of the Pith review page, Table 4, and the 7.25 argument of its
 * Fig. 2 / Theorem 1, on any tensor).
 *   x        device, [rows][cols] of `dtype` (MXATTN_BF16 / MXATTN_FP32),
 *            row-major; groups of 32 consecutive elements along each row from
 *            index 0, the tail zero-padded.  rotate = 1 Hadamard-rotates every
 *            row first exactly as mxattn_hadamard_quant_qk does (cols = 64 or
 *            128).  For V or P~ pass the key-major (transposed) matrix.
 *   qs       HOST array of nq boundaries (1 <= nq <= 64), each in [4, 8], in
 *            increasing order; each is a ceiling rule (smallest e with
 *            amax <= q 2^e).
 *   counts   device [nq] unsigned 64-bit: += the number of groups for which
 *            q_k gives the smallest squared reconstruction error (a group counts
 *            for every optimal q_k: ties are common, the error depends on q only
 *            through the exponent).
 *   sse_sums device [nq] fp64: += the summed squared error at q_k (each group's
 *            error in fp64 in index order; the sum over groups is atomic, so its
 *            last bits depend on timing).
 * Both outputs accumulate; the caller zeroes them.  Invalid arguments return
 * MXATTN_ERR_INVALID_ARG before anything is enqueued.  No counterpart on the
 * pages beyond the study it reproduces.
 */
MXATTN_API mxattn_status mxattn_qmax_sweep(const void* x, int64_t rows, int64_t cols, int dtype, int rotate,
                                           const float* qs, int nq, unsigned long long* counts,
                                           double* sse_sums, void* stream);

/*
 * Diagnostic variant of mxattn_attention_mxfp4: identical results, and the CTA
 * that owns query tile dump_qt (128 rows) of head dump_bh (index into B*H)
 * also writes its internal state to `dump` (device buffer of
 * mxattn_attention_dump_bytes(N, d) bytes, 16-byte aligned), in this order:
 *   S of key tiles 0 and 1       fp32 [2][128][64], raw Q^ K^T from the MMA
 *   P^ codes of every key tile   [ceil(N/64)][128][32] bytes, keys in order,
 *                                element 2i in the low nibble
 *   P^ scales of every key tile  [ceil(N/64)][128][2] E8M0 bytes (groups 0, 1)
 *   O~ accumulator               fp32 [128][d] before the division by l
 *   l, m                         fp32 [128] each; m = running max of
 *                                S * softmax_scale * log2(e) used for P~
 *   P~ of every key tile         fp32 [ceil(N/64)][128][64]: the unquantized
 *                                2^(S * softmax_scale * log2(e) - m) with that
 *                                tile's running max (0 for keys past N)
 *   m of every key tile          fp32 [ceil(N/64)][128], after its update
 * (the O~, l, m block starts at the next 16-byte boundary).  Used to measure
 * how many P^ codes differ from the oracle's and to study P~'s quantization
 * (per-block Qmax sweep, row-sum error decomposition); the paper has no
 * counterpart.  Full attention in MXFP4 only: opts->causal or the NVFP4
 * format return MXATTN_ERR_UNSUPPORTED.
 */
MXATTN_API size_t mxattn_attention_dump_bytes(int N, int d);
MXATTN_API mxattn_status mxattn_attention_mxfp4_dump(
    const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes, const uint8_t* k_scales,
    const uint8_t* v_codes, const uint8_t* v_scales, int B, int H, int N, int d, float softmax_scale,
    const mxattn_opts* opts, void* out, int dump_bh, int dump_qt, uint8_t* dump, void* stream);

/*
 * The whole forward pass: mxattn_hadamard_quant_qk + mxattn_quant_v into
 * the workspace, then mxattn_attention_mxfp4.  d in {64, 128}, N >= 1.
 */
MXATTN_API mxattn_status mxattn_forward(const void* q, const void* k, const void* v, int B, int H, int N,
                             int d, float softmax_scale, const mxattn_opts* opts, void* out,
                             void* stream);

/*
 * The forward pass from and to HOST memory: q_host, k_host, v_host and
 * out_host are [B][H][N][d] of opts->dtype in host memory.  The B*H heads run
 * in up to 40 chunks (independent problems): chunk c's inputs are copied to
 * the device on an internal stream while chunk c-1 computes, and its output
 * is copied back on another internal stream while chunk c+1 computes, so the
 * transfers overlap the kernels.  Even chunks compute on `stream`, odd ones
 * on a third internal stream, each with its own packed-operand buffers, so
 * that a chunk's kernels fill the SMs the previous chunk's last CTAs leave
 * idle.  Host buffers should be page-locked (cudaHostAlloc /
 * cudaHostRegister) for the copies to overlap; pageable buffers give the same
 * result without the overlap.  The workspace (device, 256-byte aligned) holds
 * mxattn_workspace_bytes_host(B, H, N, d, opts) bytes (double-buffered
 * staging and packed operands of one chunk).  Every copy and kernel is
 * ordered before the work enqueued on `stream` afterwards: synchronize
 * `stream` before reading out_host.  The first call on a device creates
 * three non-blocking streams and seven events for that device, kept until the
 * process exits; calls on one device enqueue their work one at a time (a host
 * lock).  The call allocates no device memory.  Results equal
 * mxattn_forward's bit for bit.  Errors as for mxattn_forward (a failed CUDA
 * call returns MXATTN_ERR_CUDA).  The paper has no counterpart.
 */
MXATTN_API size_t mxattn_workspace_bytes_host(int B, int H, int N, int d, const mxattn_opts* opts);
MXATTN_API mxattn_status mxattn_forward_host(const void* q_host, const void* k_host, const void* v_host, int B,
                                             int H, int N, int d, float softmax_scale, const mxattn_opts* opts,
                                             void* out_host, void* stream);

/*
 * Cross-attention (queries and keys of different lengths, e.g. video tokens
 * attending to text tokens): q and out [B][H][Nq][d], k and v [B][H][Nk][d],
 * all of opts->dtype, device, 16-byte aligned, non-causal; the same
 * rotation, quantization and PNQ loop as mxattn_forward, with the key tiles and
 * the ragged last key tile taken from Nk.  The workspace (256-byte aligned)
 * holds mxattn_workspace_bytes_cross(B, H, Nq, Nk, d, opts) bytes (0 for
 * invalid sizes); mxattn_forward_cross(.., N, N, ..) computes what
 * mxattn_forward does.  Errors as for mxattn_forward.  The pages' video models
 * use text cross-attention beside self-attention; they fix no API for it.
 */
MXATTN_API size_t mxattn_workspace_bytes_cross(int B, int H, int Nq, int Nk, int d, const mxattn_opts* opts);
MXATTN_API mxattn_status mxattn_forward_cross(const void* q, const void* k, const void* v, int B, int H, int Nq,
                                              int Nk, int d, float softmax_scale, const mxattn_opts* opts,
                                              void* out, void* stream);

/*
 * Packed batch of variable-length sequences ("varlen"): nseq self-attention
 * problems of different lengths in one call, e.g. videos of different
 * durations batched together.  Each sequence is a problem of its own, computed
 * exactly as mxattn_forward computes one head of it: its V groups of 32 keys
 * start at its first token, its ragged last tile is masked, and opts->causal
 * applies within it.  The pages fix no API for this.
 *  - q, k, v, out: TOKEN-MAJOR [T, H, d] in opts->dtype (T = total tokens,
 *    row (t, h) at element (t*H + h)*d), 16-byte aligned device pointers.
 *  - cu_seqlens: DEVICE int32 [nseq + 1], sequence s = tokens cu_seqlens[s] ..
 *    cu_seqlens[s+1]-1; it must start at 0, never decrease and end at T.
 *    Empty sequences are allowed.  Being on the device it is checked there: a
 *    table that breaks the rule makes the pass write nothing and records a
 *    status that mxattn_get_device_error reports as MXATTN_ERR_INVALID_ARG.
 *  - nseq in [1, 2^24], H in [1, 65535], d in {64, 128}.
 *  - Workspace: mxattn_workspace_bytes_varlen(nseq, H, T, d, opts) bytes
 *    (0 for invalid sizes), 256-byte aligned: status block, the sequences'
 *    tile table, then the packed operands with every sequence padded to whole
 *    128-row tiles ((T + 127*nseq)/128 tiles per head are reserved).
 *  - Four launches on `stream`: the tile table, Q/K rotation+quantization, V
 *    quantization, the attention.  Other errors as for mxattn_forward.
 */
MXATTN_API size_t mxattn_workspace_bytes_varlen(int nseq, int H, int T, int d, const mxattn_opts* opts);
MXATTN_API mxattn_status mxattn_forward_varlen(const void* q, const void* k, const void* v, const int* cu_seqlens,
                                               int nseq, int H, int T, int d, float softmax_scale,
                                               const mxattn_opts* opts, void* out, void* stream);

/*
 * mxattn_forward without a caller-provided workspace, for callers that cannot
 * allocate device memory: a process whose memory manager has already reserved
 * the GPU's memory (a cudaMalloc would fail or fragment its pool), or a plain C
 * caller without allocator plumbing.  The paper has no counterpart; this is a
 * deployment variant of the same pass.
 *  - Scratch (packed Q/K/V operands and the status block) comes from a fixed
 *    64 MiB array inside the library; every GPU that loads the library holds it
 *    until the process exits.  Problems whose mxattn_workspace_bytes() exceeds
 *    64 MiB (at d = 128, about 300k query rows summed over B*H) are rejected
 *    with MXATTN_ERR_WORKSPACE before anything is enqueued.
 *  - opts->workspace and opts->workspace_bytes are ignored.  No memory is
 *    allocated or freed by this call.
 *  - The first call on a device looks up the array's device address (with that
 *    device current); make that first call before any stream capture.
 *  - All calls share the one array: calls that may overlap on the GPU (other
 *    streams, other host threads) race and corrupt each other's results;
 *    serialize them.  The status block is cleared at the start of every call,
 *    so a bounded-wait expiry is not reported through mxattn_get_device_error.
 *  - q, k, v, out: as mxattn_forward, on the current device.
 */
MXATTN_API mxattn_status mxattn_forward_noalloc(const void* q, const void* k, const void* v, int B, int H,
                                                int N, int d, float softmax_scale, const mxattn_opts* opts,
                                                void* out, void* stream);

/*
 * Synchronize `stream`, read the workspace status block and clear it.
 * Returns MXATTN_ERR_TIMEOUT if a kernel gave up on a bounded wait since the
 * last call (its output is then undefined), MXATTN_ERR_INVALID_ARG if a
 * varlen call found its cu_seqlens table invalid (nothing was written),
 * MXATTN_OK otherwise.
 */
MXATTN_API mxattn_status mxattn_get_device_error(const mxattn_opts* opts, void* stream);

/* Static string naming a status code. */
MXATTN_API const char* mxattn_status_string(mxattn_status status);

/*
 * Dense FP4 tensor-core throughput probe (not part of the method): `ctas`
 * CTAs each issue `iters` back-to-back tcgen05 kind::mxf4 block-scaled MMAs
 * of shape M=128 x n x K=64 from shared memory into tensor memory.
 * n in {64, 128, 256}.  The caller times the launch; flops = ctas * iters *
 * 2 * 128 * n * 64.
 */
MXATTN_API mxattn_status mxattn_fp4_mma_probe(int ctas, int iters, int n, void* stream);

/*
 * Arithmetic probe (a diagnostic, not part of the method; the paper has no
 * counterpart): evaluates one of the attention kernels' arithmetic shortcuts
 * element-wise on n device floats `in`, writing device array `out`, so that
 * tests can hold it against its definition.  The scale rule is opts'.
 *   MXATTN_PROBE_EXP2_POLY            out float[n]: the FMA-pipe exp2
 *       polynomial of the 64-key kernel at in[i]
 *   MXATTN_PROBE_EXP2_MUFU            out float[n]: ex2.approx(in[i])
 *   MXATTN_PROBE_E2M1_OF_EXP2_STANDIN out uint8[n]: the E2M1 code (round to
 *       nearest even, saturating) that the 128-key kernel's FMA-pipe stand-in
 *       for 2^u gives at u = in[i] (exact in code space by design)
 *   MXATTN_PROBE_E2M1_OF_EXP2_MUFU    out uint8[n]: the E2M1 code of
 *       ex2.approx(in[i])
 *   MXATTN_PROBE_SCALE_EXP_LOG2       out int32[n]: the shared exponent e the
 *       softmax computes for a group maximum 2^t given as t = in[i]
 *   MXATTN_PROBE_SCALE_EXP            out int32[n]: the shared exponent e the
 *       quantizers compute for amax = in[i] (exact integer rule)
 * in 4-byte aligned; out 4-byte aligned for the float and int32 outputs.
 * Invalid op, sizes or options -> MXATTN_ERR_INVALID_ARG, nothing enqueued.
 */
enum {
  MXATTN_PROBE_EXP2_POLY = 0,
  MXATTN_PROBE_EXP2_MUFU = 1,
  MXATTN_PROBE_E2M1_OF_EXP2_STANDIN = 2,
  MXATTN_PROBE_E2M1_OF_EXP2_MUFU = 3,
  MXATTN_PROBE_SCALE_EXP_LOG2 = 4,
  MXATTN_PROBE_SCALE_EXP = 5
};
MXATTN_API mxattn_status mxattn_arith_probe(int op, const float* in, int64_t n, const mxattn_opts* opts, void* out,
                                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MXATTN_H_ */
