/*
 * nq.h -- C ABI of libnq: the forward pass of a linear layer whose weight is stored as a
 * low-rank binary factorisation,
 *
 *     W ~= diag(s1) . U . V^T . diag(s2),   U in {+1,-1}^{m x r},  V in {+1,-1}^{n x r},
 *     y  = s1 (.) ( U . ( V^T . ( s2 (.) x ) ) ),
 *
 * with U and V stored one bit per entry and s1 (m), s2 (n) fp16 scale vectors.
 * The method is NanoQuant's (hardwired.dev, "NanoQuant jednoduse: 70B model na herni
 * grafice", section "Jak NanoQuant funguje": the weight matrix as a product of +1/-1
 * matrices and diagonal scaling vectors, r*(m+n) binary values plus the scales;
 * rapidrecap.app, "Nanoquant: Efficient Sub-1-Bit Quantization of Large Language
 * Models", section "Quantization Technique": binary U and V plus scaling factors,
 * evaluated by custom CUDA kernels; hardwired.dev section "Cisla": binary GEMV/GEMM
 * kernels).  The pages publish no kernel and no interface; this ABI is this library's.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Plain pointers and sizes; no ownership transfer: every buffer is owned by the caller.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream.
 *  - Return value: an nq_status (0 = NQ_OK, negative = error).  Argument errors are
 *    detected on the host before anything is enqueued; in that case nothing is launched
 *    and no output is written.
 *  - Stored form of a sign matrix ("packed"): row-major rows of ceil(cols/32) uint32
 *    words; bit b of word w of a row is the entry in column 32*w + b; bit 1 = +1,
 *    bit 0 = -1; unused high bits of a partial last word are 0.
 *      Upk: U as m rows of r/32 words         (row i = U[i][0..r))
 *      Vpk: V^T as r rows of n/32 words       (row k = V[0..n)[k])
 *  - x, s1, s2 hold IEEE bit patterns: x bfloat16, s1 and s2 binary16 (fp16).
 *  - "Device memory" means memory of the device current on the calling thread, or managed
 *    memory; device memory of another GPU is refused with NQ_ERR_PTRKIND before anything
 *    is enqueued (a kernel given it without peer access would fault).
 *  - The library keeps one workspace per device (intermediate t = V^T (s2 (.) x) and
 *    a few counters).  It is allocated on the first call on a device and grown when a
 *    larger shape arrives; call nq_workspace_reserve() beforehand to keep allocation out
 *    of a CUDA-graph capture.  Calls that use the same device's workspace must not run
 *    concurrently on different streams.
 */
#ifndef NQ_H_
#define NQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NQ_OK = 0,
    NQ_ERR_NULL = -1,      /* a required pointer is NULL */
    NQ_ERR_SHAPE = -2,     /* a size is out of range or not a supported multiple */
    NQ_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned */
    NQ_ERR_BATCH = -4,     /* batch < 0 */
    NQ_ERR_VALUE = -5,     /* an input value is outside its domain (e.g. a sign of 2) */
    NQ_ERR_CUDA = -6,      /* a CUDA runtime/driver call or a launch failed */
    NQ_ERR_TIMEOUT = -7,   /* a bounded device-side wait gave up */
    NQ_ERR_NOMEM = -8,     /* workspace allocation failed */
    NQ_ERR_PTRKIND = -9,   /* pointers of mixed or unsupported memory kinds, or device
                              memory of a GPU other than the current one */
    NQ_ERR_NOALLOC_LIMIT = -10 /* size beyond nq_lowrank_linear_fwd_noalloc's fixed scratch */
} nq_status;

/* Largest decode batch: calls with 1 <= batch <= NQ_DECODE_MAX_BATCH run the two-stage
 * binary GEMV; larger batches run the tensor-core path. */
#define NQ_DECODE_MAX_BATCH 8

/*
 * nq_pack_signs -- store a sign matrix one bit per entry (the sign projection of the
 * ADMM step, hardwired.dev section "Krok 2", followed by the one-bit storage of section
 * "Jak NanoQuant funguje").
 *   signs : rows x cols int8, row-major; each entry -1, 0 or +1 (0 is stored as +1).
 *   out   : rows x ceil(cols/32) uint32 (layout above).
 *   rows, cols >= 0; rows*cols == 0 is a no-op returning NQ_OK.
 * Both pointers on the device: a kernel runs on `stream`, then the call synchronises
 * `stream` to read back the value check (packing is an offline step).  Both pointers in
 * host memory: packed on the calling thread, `stream` unused.  Mixed: NQ_ERR_PTRKIND.
 * An entry outside {-1, 0, +1} returns NQ_ERR_VALUE; `out` is then unspecified.
 */
int nq_pack_signs(const int8_t* signs, int64_t rows, int64_t cols, uint32_t* out, void* stream);

/*
 * nq_unpack_signs -- inverse of nq_pack_signs: rows x cols int8 in {-1, +1}.
 * Same pointer-kind rules; the device path does not synchronise.
 */
int nq_unpack_signs(const uint32_t* packed, int64_t rows, int64_t cols, int8_t* out, void* stream);

/*
 * nq_lowrank_linear_fwd -- y = s1 (.) (U (V^T (s2 (.) x))) for `batch` tokens.
 *   x    : batch x n bfloat16, row-major (one token per row)
 *   Upk  : m x (r/32) uint32, device memory
 *   Vpk  : r x (n/32) uint32, device memory
 *   s1   : m fp16, device memory;  s2 : n fp16, device memory
 *   y    : batch x m float32, row-major (written)
 *   m, n, r : positive multiples of 128, each at most 1<<20
 *   batch   : >= 0; 0 is a no-op returning NQ_OK
 * x and y may be device memory, or host memory (pageable or pinned): host x is brought to
 * the device on `stream` first (pinned x by a copy kernel that reads it through its device
 * address, pageable x by a copy), pinned host y is written by the kernels directly and
 * pageable host y copied back; with any host buffer the call then synchronises `stream`
 * before returning.  Device buffers are used asynchronously on `stream`.
 * A synchronising call whose host buffers are all pinned is replayed from a CUDA graph
 * once the identical call (same pointers, sizes and library scratch) has been made before:
 * its second occurrence captures the launches into a graph that the library keeps (up to
 * 32 per device, least recently used dropped first), later ones launch that graph, which
 * costs less host time than the separate launches.  The graph reads the buffers' contents
 * at the time of each call, like a direct launch.  Not on a stream under capture.
 * Every pointer must be 16-byte aligned.
 * Path: batch <= NQ_DECODE_MAX_BATCH runs the decode path (two binary GEMV stages on the
 * CUDA cores and integer tensor-core instructions, t kept in the workspace); larger
 * batches run the prefill path (two tcgen05 tensor-core GEMMs with the +1/-1 operands
 * expanded on chip, fp16 operands, fp32 accumulation).
 * Accuracy: max|y - y_exact| / max|y_exact| <= 2e-3, over the call and over each token
 * alone (each token's error against its own largest output), for finite inputs in these
 * ranges.  Decode: per token the largest |s2_j x_j| of every 1024-column chunk in
 * [2^-90, 2^100] (each chunk is quantised to 14 bits under its own power of two, t under one
 * per token).  Prefill: per token L = sum_j |s2_j x_j| in [2^-95, 2^126] (x' and T carry a
 * power of two per token that keeps them below 2^15, inside fp16's normal range).
 * Tested against an fp64 reference with N(0,1) activations, three outlier channels per
 * 1024 columns at 1e2..1e4, magnitudes 2^-20..2^10 inside every chunk, tokens of 1e-20 to
 * 1e20 in one call, |s2_j x_j| near 6e4 and near 2e-8, and zero tokens (exact zeros out).
 * Weights (Upk, Vpk, s1, s2) may be read before the work enqueued earlier on `stream`
 * has finished (programmatic dependent launch), so they must not be produced by the
 * kernel enqueued immediately before this call on the same stream; x may be.
 */
int nq_lowrank_linear_fwd(const void* x, const uint32_t* Upk, const uint32_t* Vpk,
                          const void* s1, const void* s2, int64_t m, int64_t n, int64_t r,
                          int64_t batch, float* y, void* stream);

/*
 * nq_transpose_signs -- the transpose of a packed sign matrix: `packed` holds rows x cols
 * entries as rows x ceil(cols/32) uint32 (the layout of nq_pack_signs), `out` receives the
 * cols x rows transpose as cols x ceil(rows/32) uint32 in the same layout (unused high bits
 * of each row's last word zero).  rows, cols >= 0; rows*cols == 0 is a no-op returning
 * NQ_OK.  Both pointers on the device (a kernel on `stream`, no synchronisation) or both
 * in host memory (on the calling thread); mixed: NQ_ERR_PTRKIND.  Used to give the
 * backward pass its packings: UpkT = transpose of Upk (m x r -> r x m), VpkT = transpose of
 * Vpk (r x n -> n x r).  `out` must not overlap `packed`.
 */
int nq_transpose_signs(const uint32_t* packed, int64_t rows, int64_t cols, uint32_t* out, void* stream);

/*
 * nq_lowrank_linear_bwd_input -- the gradient of the layer's output with respect to its
 * input, dx = W^T dy = s2 (.) (V (U^T (s1 (.) dy))), for `batch` tokens: the step of the
 * straight-through refinement of the factorised components (hardwired.dev, "Krok 3")
 * that passes the gradient on to the layer before.
 *   dy   : batch x m bfloat16, row-major (one token per row)
 *   UpkT : r x (m/32) uint32, device memory (rows of U^T: nq_transpose_signs(Upk, m, r))
 *   VpkT : n x (r/32) uint32, device memory (rows of V: nq_transpose_signs(Vpk, r, n))
 *   s1   : m fp16, s2 : n fp16, device memory (the layer's scales)
 *   dx   : batch x n float32, row-major (written)
 * It is the forward pass of the layer with the roles of the factors exchanged (U' = V,
 * V' = U, s1' = s2, s2' = s1, m' = n, n' = m), so every rule, path and accuracy statement
 * of nq_lowrank_linear_fwd applies with those names; dy and dx may be host memory as x
 * and y there.
 */
int nq_lowrank_linear_bwd_input(const void* dy, const uint32_t* UpkT, const uint32_t* VpkT, const void* s1,
                                const void* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* dx,
                                void* stream);

/*
 * nq_lowrank_linear_bwd_scales -- the gradients with respect to the two scale vectors,
 * for `batch` tokens of input x and output gradient dy (the refinement step tunes the
 * scales with the factors, hardwired.dev "Krok 3"):
 *     ds1_i = sum_b dy[b][i] * (U (V^T (s2 (.) x[b])))_i
 *     ds2_j = sum_b x[b][j]  * (V (U^T (s1 (.) dy[b])))_j
 *   x    : batch x n bfloat16;  dy : batch x m bfloat16
 *   Upk, Vpk   : the forward packings;  UpkT, VpkT : their transposes (nq_transpose_signs)
 *   s1 : m fp16;  s2 : n fp16
 *   ds1 : m float32, ds2 : n float32 (written; either may be NULL to skip it)
 * Every pointer in device memory, 16-byte aligned (else NQ_ERR_PTRKIND / NQ_ERR_ALIGN);
 * shapes as nq_lowrank_linear_fwd; batch 0 writes zeros.  Each gradient is the layer
 * evaluated without one scale (the forward pass, or the input gradient, with that scale
 * set to 1, through the decode or prefill kernels) followed by a per-column dot product
 * over the tokens: 64-token chunks each summed in token order, then the chunks' sums in
 * chunk order (a fixed order, so repeated calls agree bit for bit).  Accuracy: each term
 * carries the error
 * of that evaluation, |error of ds1_i| <= 2e-3 * sum_b |dy[b][i]| * max_i' |z[b][i']|.
 * Uses the workspace (not safe for concurrent calls on different streams); asynchronous
 * on `stream`, except that the first call of a size allocates scratch.
 */
int nq_lowrank_linear_bwd_scales(const void* x, const void* dy, const uint32_t* Upk, const uint32_t* Vpk,
                                 const uint32_t* UpkT, const uint32_t* VpkT, const void* s1, const void* s2,
                                 int64_t m, int64_t n, int64_t r, int64_t batch, float* ds1, float* ds2,
                                 void* stream);

/*
 * nq_lowrank_linear_bwd_factors -- the straight-through gradients of the two factors (the
 * refinement step passes the gradient of the sign function as the identity, hardwired.dev
 * "Krok 3", so these are the gradients with respect to the latent real-valued factors):
 *     dU[i][k] = s1_i * sum_b dy[b][i] * t[b][k],   t = V^T (s2 (.) x)
 *     dV[j][k] = s2_j * sum_b x[b][j]  * u[b][k],   u = U^T (s1 (.) dy)
 *   x  : batch x n bfloat16;  dy : batch x m bfloat16
 *   Vpk : r x (n/32) (the forward packing of V^T);  UpkT : r x (m/32) (transpose of Upk)
 *   s1 : m fp16;  s2 : n fp16
 *   dU : m x r float32, dV : n x r float32, row-major (written; either may be NULL)
 * Every pointer in device memory, 16-byte aligned; shapes as nq_lowrank_linear_fwd; batch 0
 * writes zeros.  Below 64 tokens, t and u come from the decode path's first stage (up to 8
 * tokens per launch) and the sums over the tokens from a tiled fp32 kernel in token order.
 * From 64 tokens, t and u come from the prefill path's first GEMM and the sums from a
 * tensor-core GEMM: dy (or x) in bf16 against t split into two bf16 parts (t = hi + lo,
 * the pair exact to 2^-16 relative), accumulated in fp32 on the tensor cores; the order is
 * fixed by the tile shapes, so repeated calls agree bit for bit.  Accuracy, both routes:
 * |error of dU[i][k]| <= 2e-3 * |s1_i| * sum_b |dy[b][i]| * max_k' |t[b][k']| (likewise
 * dV).  Uses the workspace.
 */
int nq_lowrank_linear_bwd_factors(const void* x, const void* dy, const uint32_t* Vpk, const uint32_t* UpkT,
                                  const void* s1, const void* s2, int64_t m, int64_t n, int64_t r, int64_t batch,
                                  float* dU, float* dV, void* stream);

/* One factorised layer of a grouped call (same meaning and rules as the arguments of
 * nq_lowrank_linear_fwd; every pointer in device memory, 16-byte aligned). */
typedef struct nq_linear_desc {
    const void* x;          /* batch x n bfloat16 */
    const uint32_t* Upk;    /* m x (r/32) */
    const uint32_t* Vpk;    /* r x (n/32) */
    const void* s1;         /* m fp16 */
    const void* s2;         /* n fp16 */
    float* y;               /* batch x m float32 (written) */
    int64_t m, n, r;
} nq_linear_desc;

/*
 * nq_lowrank_linear_fwd_grouped -- `count` independent factorised layers with the same
 * batch, e.g. the projections of one transformer block that read the same or different
 * activations.  The result of every layer equals nq_lowrank_linear_fwd on it; the
 * decode path (batch <= NQ_DECODE_MAX_BATCH) runs up to 16 layers per launch pair, so
 * small layers share the launch and dependency latency.  With more tokens (up to 64) and
 * more than one layer, the call runs the decode path over token chunks of at most
 * NQ_DECODE_MAX_BATCH instead of each layer's prefill GEMMs one after another when a cost
 * estimate (fitted to B200 timings) finds that faster: several layers and a few dozen
 * tokens, e.g. the seven Llama-2-7B-shaped projections up to 48 tokens.  Each token's
 * result is then that of the decode path, within the same accuracy bound.  No layer's y may overlap
 * another layer's inputs.  Argument checks as nq_lowrank_linear_fwd, plus count >= 0
 * (0 is a no-op) and `layers` non-NULL.  Weights (Upk, Vpk, s1, s2) must be device memory
 * (else NQ_ERR_PTRKIND).  Each layer's x and y may be device or host memory, handled as
 * in nq_lowrank_linear_fwd (pinned x gathered by one kernel for all layers, pinned y
 * written directly, pageable buffers copied); with any host buffer the call synchronises
 * `stream` before returning (and, with only pinned host buffers, is replayed from a kept
 * CUDA graph when repeated, as nq_lowrank_linear_fwd), with only device buffers it is
 * asynchronous.
 */
int nq_lowrank_linear_fwd_grouped(const nq_linear_desc* layers, int count, int64_t batch, void* stream);

/*
 * Helpers for running factorised layers one after another (a decode chain).  A decoder
 * runs its quantised linear layers in sequence (hardwired.dev section "Cisla": decode
 * tokens/s of a whole quantised model); the pages print nothing about what sits between
 * the layers, so these are the library's own glue, not steps of the method: each
 * forward call takes bfloat16 x and returns fp32 y, and these turn one layer's y into the
 * next layer's x.  Both pointers in device memory, 16-byte aligned; the kernels are
 * asynchronous on `stream` and, like the forward call, may start before the kernel
 * enqueued just before them has finished: they read `src` only after it has.
 *
 * nq_cast_f32_to_bf16 -- dst[i] = bf16(src[i]) for 0 <= i < count, round to nearest,
 *   ties to even (overflow to infinity, NaN stays NaN).  count >= 0 (0 is a no-op).
 *   dst: count bfloat16 (uint16 patterns), written; it must not overlap src.
 */
int nq_cast_f32_to_bf16(const float* src, int64_t count, void* dst, void* stream);

/*
 * nq_rms_normalize_bf16 -- re-normalise each row to unit root-mean-square:
 *   dst[i][j] = bf16( src[i][j] / sqrt( (1/cols) * sum_j src[i][j]^2 ) ),
 *   computed in fp32 (sum of squares, one reciprocal square root per row, one product
 *   per element) and rounded to nearest, ties to even.  A row whose sum of squares is 0
 *   is rounded unchanged.  src: rows x cols float32 row-major; dst: rows x cols bfloat16,
 *   written, not overlapping src.  rows >= 0 (0 is a no-op), cols >= 1.
 */
int nq_rms_normalize_bf16(const float* src, int64_t rows, int64_t cols, void* dst, void* stream);

/* A layer of nq_lowrank_linear_fwd_grouped_ex: the layer plus two optional outputs that
 * feed the next layer of a chain (see nq_cast_f32_to_bf16 / nq_rms_normalize_bf16 above;
 * like them, these have no counterpart in the NanoQuant pages). */
typedef struct nq_linear_desc_ex {
    nq_linear_desc base;     /* the layer, as for nq_lowrank_linear_fwd_grouped */
    void* y_bf16;            /* NULL, or batch x m bfloat16 written with bf16(y) */
    void* y_rmsnorm_bf16;    /* NULL, or batch x m bfloat16 written with
                              * bf16(y[b][i] / sqrt((1/m) sum_i y[b][i]^2)) per token b */
} nq_linear_desc_ex;

/*
 * nq_lowrank_linear_fwd_grouped_ex -- nq_lowrank_linear_fwd_grouped, plus per layer the
 * optional bfloat16 copies of y that the next layer of a decode chain reads.  y is always
 * written.  y_bf16 equals nq_cast_f32_to_bf16 of y bit for bit; y_rmsnorm_bf16 equals
 * nq_rms_normalize_bf16 of y (batch rows of m) up to the order of the fp32 sum of squares.
 * On the decode path both are produced by the forward's own kernels (no extra launch); on
 * the prefill path by the stand-alone kernels after the layer.  Optional pointers are
 * device memory, 16-byte aligned, and overlap no other buffer of the call.  Errors as
 * nq_lowrank_linear_fwd_grouped, except that every buffer, x and y included, must be
 * device memory (else NQ_ERR_PTRKIND).
 */
int nq_lowrank_linear_fwd_grouped_ex(const nq_linear_desc_ex* layers, int count, int64_t batch, void* stream);

/*
 * nq_lowrank_linear_fwd_envelope -- the rank-l envelope variant of the layer (MDBF-style
 * scaling; hardwired.dev section "Kontext: co existuje kolem": MDBF replaces the simple
 * scaling of the binary factorisation with a rank-l envelope, since under the simple
 * scaling all rank components share one magnitude profile).  The library's reading:
 *     W = (sum_{q<l} a_q b_q^T) (.) (U V^T),   y = sum_{q<l} a_q (.) (U (V^T (b_q (.) x))),
 * l = 1 being nq_lowrank_linear_fwd with s1 = a_0, s2 = b_0 (bit for bit the same result).
 *   a : l x m fp16 (row q = a_q);  b : l x n fp16 (row q = b_q);  1 <= l <= 16
 *   x, Upk, Vpk, y, m, n, r, batch: as nq_lowrank_linear_fwd.  Every pointer device memory
 *   of the current device (else NQ_ERR_PTRKIND), 16-byte aligned.
 * The l terms run as one grouped call (layers sharing U and V: one decode launch pair for
 * up to 8 tokens, or each term's prefill GEMMs), term 0 into y and the others into library
 * scratch (allocated on first use of a size), then one kernel adds terms 1 .. l-1 to y in
 * increasing q.  Asynchronous on `stream`; uses the workspace like the forward.
 * Accuracy: each term within the forward's bound, so max|y - y_exact| <= 2e-3 * sum_q
 * max|term_q| (tested: within 2e-3 of max|y_exact|, globally and per token, for l = 2, 4).
 */
int nq_lowrank_linear_fwd_envelope(const void* x, const uint32_t* Upk, const uint32_t* Vpk, const void* a,
                                   const void* b, int64_t l, int64_t m, int64_t n, int64_t r, int64_t batch,
                                   float* y, void* stream);

/* Bits per weight of the envelope variant: (r*(m+n) + 16*l*(m+n)) / (m*n); -1.0 if any
 * argument is <= 0.  Equals nq_bits_per_weight for l = 1. */
double nq_bits_per_weight_envelope(int64_t m, int64_t n, int64_t r, int64_t l);

/* Limits of nq_lowrank_linear_fwd_noalloc. */
#define NQ_NOALLOC_MAX_RANK 4096
#define NQ_NOALLOC_MAX_BATCH NQ_DECODE_MAX_BATCH

/*
 * nq_lowrank_linear_fwd_noalloc -- the decode path of nq_lowrank_linear_fwd for callers
 * that cannot allocate device memory when they run a layer: an inference engine that
 * reserved its memory pool at start-up (a later cudaMalloc competes with that pool and can
 * fail in the middle of a request), or a host framework that owns the allocator (a side
 * allocation escapes its accounting).  It has no counterpart in the NanoQuant pages: it is
 * a property of this library, not of the method.
 *   Same arguments, layout and result as nq_lowrank_linear_fwd, restricted to
 *   1 <= batch <= NQ_NOALLOC_MAX_BATCH and r <= NQ_NOALLOC_MAX_RANK (larger sizes return
 *   NQ_ERR_NOALLOC_LIMIT; batch 0 is a no-op).  Every pointer must be device memory of the
 *   current device (else NQ_ERR_PTRKIND, before anything is enqueued).
 *   Scratch: a fixed array of 1,180,800 bytes (1.18 MB) compiled into the library's device
 *   code, held by every GPU that loads the library until the process exits.  The call
 *   allocates and frees nothing, on the host or the device.
 *   The first call on each device resolves the array's device address (with that device
 *   current); make that first call before any stream capture that includes this entry.
 *   All calls share the one array and each call overwrites it: calls whose kernels could
 *   overlap on the GPU (other streams, other host threads on the same device) race, and
 *   must be ordered by the caller.
 */
int nq_lowrank_linear_fwd_noalloc(const void* x, const uint32_t* Upk, const uint32_t* Vpk,
                                  const void* s1, const void* s2, int64_t m, int64_t n, int64_t r,
                                  int64_t batch, float* y, void* stream);

/*
 * LB-ADMM initialiser of the binary factorisation (hardwired.dev, "NanoQuant jednoduse",
 * section "Trikrokovy pipeline", step 2 "Inicializace binarni faktorizace (LB-ADMM)": ADMM
 * alternating a closed-form least-squares solve for the continuous parameters with a
 * projection onto the binary constraint by the sign operation, followed by magnitude
 * balancing of the scales).  The pages give no formula; the library's reading:
 *   W ~= A B^T with latent A (m x r), B (n x r) constrained to row-scaled sign matrices
 *   Z = diag(s) S, S in {+1,-1}; scaled duals L_A, L_B; iteration k with lam_k = lam0*growth^k:
 *     rho_A = lam_k tr(B^T B)/r;  A = (W B + rho_A (Z_A - L_A)) (B^T B + rho_A I)^-1;
 *     Z_A = Pi(A + L_A) (per row: signs, sign(0) = +1, and the scale mean |row|);
 *     L_A = L_A + A - Z_A;  then the same for B with W^T and the new A.
 *   Start: block power iteration from Omega (n x r): Q = orth(W Omega), power_iters times
 *   Q = orth(W (W^T Q)), orth by Cholesky-QR; A = Q, B = W^T Q, each column pair rescaled
 *   to equal norms; Z = Pi(A), Pi(B); L = 0.
 *   Result: U = signs of Z_A, V = signs of Z_B; s1 = c s_A, s2 = s_B / c with
 *   c = sqrt(rms(s_B)/rms(s_A)) (both scale vectors get the same root-mean-square).
 * Common rules: W is m x n bfloat16, row-major, device memory; every matrix is row-major
 * fp32 device memory of the current device, 16-byte aligned (else NQ_ERR_ALIGN /
 * NQ_ERR_PTRKIND); m, n, r positive multiples of 128 with r <= min(m, n) and r <= 16384
 * (else NQ_ERR_SHAPE).  The calls allocate their own scratch (cudaMalloc) and synchronise
 * `stream` before returning (an offline step).  A Cholesky pivot that is not positive in
 * fp32 (a start W Omega of column rank below r, or an ill-conditioned system) returns
 * NQ_ERR_VALUE; the outputs are then unspecified.  Deterministic: every sum runs in a
 * fixed order.  Arithmetic in fp32 (W read exactly from bf16), reductions of norms in fp64;
 * the iterations' products W B and W^T A run on the tensor cores with W in bf16 and the
 * fp32 factor as the sum of three bf16 parts (fp32's precision), accumulated in fp32 (the
 * iterating calls hold the split factor in their scratch: 6 max(m, n) r bytes more).  A
 * bounded wait that gives up returns NQ_ERR_TIMEOUT.
 */

/*
 * nq_admm_init -- the start: A, B (latent, m x r and n x r), Z_A, Z_B (their projections),
 * L_A, L_B (set to zero), s_A (m), s_B (n) (the projections' row scales), all written.
 * Omega: n x r fp32, the caller's start block (e.g. Gaussian); 0 <= power_iters <= 64.
 */
int nq_admm_init(const void* W, int64_t m, int64_t n, int64_t r, const float* Omega, int power_iters, float* A,
                 float* B, float* ZA, float* ZB, float* LA, float* LB, float* sA, float* sB, void* stream);

/*
 * nq_admm_iterate -- `iters` ADMM iterations on the caller's state (read and updated in
 * place: A, B, Z_A, Z_B, L_A, L_B, s_A, s_B as written by nq_admm_init), with
 * lam_k = lam0 * growth^k for k = 0 .. iters-1.  lam0 > 0, growth > 0, iters >= 0.
 */
int nq_admm_iterate(const void* W, int64_t m, int64_t n, int64_t r, float* A, float* B, float* ZA, float* ZB,
                    float* LA, float* LB, float* sA, float* sB, int iters, double lam0, double growth, void* stream);

/*
 * nq_admm_factorize -- the whole initialiser: start, `iters` iterations, magnitude
 * balancing, and the stored form the forward pass reads:
 *   Upk : m x (r/32) uint32 (U, the layout of nq_pack_signs);  Vpk : r x (n/32) uint32 (V^T)
 *   s1  : m fp16;  s2 : n fp16
 *   rel_err : NULL, or host memory receiving ||W - diag(s1) U V^T diag(s2)||_F / ||W||_F
 *             computed with the stored fp16 scales (sums of squares in fp64).
 * Typical lam0 = 0.2, growth = 1.05, power_iters = 1, iters = 40 (the values the library's
 * tests and benchmark use).
 */
int nq_admm_factorize(const void* W, int64_t m, int64_t n, int64_t r, const float* Omega, int power_iters, int iters,
                      double lam0, double growth, uint32_t* Upk, uint32_t* Vpk, void* s1, void* s2, double* rel_err,
                      void* stream);

/*
 * nq_bits_per_weight -- storage cost of the factorised layer in bits per weight of the
 * dense m x n matrix it replaces: (r*(m+n) + 16*(m+n)) / (m*n)  (hardwired.dev sections
 * "Jak NanoQuant funguje" and "Co znamena sub-1-bit").  -1.0 if any argument is <= 0.
 */
double nq_bits_per_weight(int64_t m, int64_t n, int64_t r);

/* A static, human-readable name for a status code. */
const char* nq_status_string(int status);

/*
 * nq_workspace_reserve -- allocate (or grow) the current device's workspace so that
 * later calls with these or smaller sizes allocate nothing.  Synchronises the device.
 */
int nq_workspace_reserve(int64_t m, int64_t n, int64_t r, int64_t batch);

/*
 * nq_device_status -- synchronise `stream`, then read and clear the current device's
 * status word, in which kernels record a bounded device-side wait that gave up.
 * Returns NQ_OK, NQ_ERR_TIMEOUT, or NQ_ERR_CUDA if the synchronisation itself failed.
 */
int nq_device_status(void* stream);

/*
 * nq_selftest_wait_timeout -- exercise the failure path of the device-side waits: a kernel
 * runs the same bounded wait the tensor-core kernels use, on a barrier that nothing ever
 * arrives on, gives up after `limit_ns` nanoseconds of GPU time and records NQ_ERR_TIMEOUT
 * in the device status word.  The next nq_device_status then returns NQ_ERR_TIMEOUT (and
 * clears it); the device stays usable.  No counterpart in the pages: a property of this
 * library.  1000 <= limit_ns <= 1e10, else NQ_ERR_VALUE.  Asynchronous on `stream`.
 */
int nq_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int nq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NQ_H_ */
