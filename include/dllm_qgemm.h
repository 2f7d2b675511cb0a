/*
 * dllm_qgemm — quantized projection GEMM of a diffusion-LLM denoising step, for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (mojo-dllm Architecture page, "A forward pass", steps 2 and 4, and
 * "Source map", kernels/packed.mojo, kernels/qgemm.mojo and gpu/kernels.mojo rows):
 * every projection of every layer multiplies GGUF Q4_K or Q6_K super-block weights
 * by activations quantized to int8 with one f32 scale per 256 elements; the
 * activation is quantized once and reused by the Q, K and V projections (and once
 * for gate and up); the output projection runs only on the canvas rows whose logits
 * the sampler needs.
 *
 *   out[i][n] = sum_k w[n][k] * a[row(i)][k]
 *   w = d*sc_j*q - dmin*m_j   (Q4_K, 8 sub-blocks of 32, q in 0..15, 6-bit sc, m)
 *   w = d*sc_j*(q - 32)       (Q6_K, 16 sub-blocks of 16, q in 0..63, int8 sc)
 *   a = scale[m][k/256] * qa  (qa int8 in [-127, 127])
 *
 * Integer parts are exact (int32 tensor-core accumulation per super-block); the
 * per-super-block combine with d and the activation scale is f32.  The Q4_K min term
 * (dmin * m_j times the scaled activation sums) runs on the tf32 tensor cores: the
 * hi + lo operand splits lose at most 2^-21 of each product's magnitude, and its f32
 * accumulation over a work unit's K/32 sub-block steps adds at most (K/32) * 2^-24 of
 * the running sum of magnitudes (2^-17 at K = 4096); both stay inside the tolerance
 * max(1e-5 |ref|, 1e-6 * sum|terms|), and the tests run the worst case (every term of
 * one sign, every m = 63, saturated activations) at K = 512, 3584 and 4096.
 *
 * Conventions for every call:
 *   - Device pointers unless stated otherwise; the caller allocates and owns every
 *     buffer.  Calls are asynchronous on `stream` and allocate nothing.
 *   - Returns DLLM_OK (0) or a negative DLLM_ERR_* code.  Argument errors are found
 *     on the host before anything is launched.  Errors found on the device (a row
 *     index out of range, a bounded wait that ran out) set a per-device error word
 *     that dllm_get_device_status() reports and clears; the kernel never traps.
 *   - dllm_quantize_act, dllm_rmsnorm_quantize, dllm_swiglu_quantize, dllm_qgemm and
 *     dllm_qkv_qgemm launch their kernels with programmatic dependent launch: a kernel may start while the previous kernel on
 *     the stream is finishing, and waits on the device for it to complete before
 *     touching any memory that kernel can write.  Before that wait the GEMM only
 *     prefetches its first weight tiles into L2, which is always safe.  Stream order
 *     is preserved as usual.
 *   - N must be a multiple of 128 and K a multiple of 256.  Device pointers must be
 *     16-byte aligned.
 *   - Inputs must be finite.
 */
#ifndef DLLM_QGEMM_H
#define DLLM_QGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dllm_stream_t; /* a cudaStream_t; NULL = legacy default stream */

/* GGML type ids of the weight formats.  Q5_K (mojo-dllm Architecture page, "Source map",
 * quant/kquants.mojo row) runs on the Q4_K kernel in an exact split form: dllm_repack_q5k
 * turns each 176-byte Q5_K super-block into two Q4_K-form super-blocks of a matrix twice
 * as wide, the low nibbles (d, dmin, the same scales) and the fifth bits as 0/1 nibbles
 * (16*d, dmin 0, the same scales), since d*sc*q - dmin*m = (d*sc*q4 - dmin*m) +
 * (16d)*sc*b exactly, provided 16 d is a finite f16 (|d| < 4096; GGUF scales are many
 * orders of magnitude smaller).  It keeps 2 x 144 bytes per 256 weights resident (9 bits per
 * weight, 1.64 x the GGUF size) and streams them at the Q4_K kernel's rate.
 * Q8_0 (the same row) has a kernel of its own: 32-weight blocks, each with an f16 scale d
 * (w = d*q, q int8); every block's integer dot product is one int8 MMA K step into an
 * accumulator of its own, combined in f32 as da * sum_b d_b * dot_b. */
typedef enum { DLLM_Q8_0 = 8, DLLM_Q4_K = 12, DLLM_Q5_K = 13, DLLM_Q6_K = 14 } dllm_qtype;

enum {
    DLLM_OK = 0,
    DLLM_ERR_ARG = -1,         /* null pointer, bad size, K % 256, N % 128, ld too small, ... */
    DLLM_ERR_ALIGN = -2,       /* a pointer or leading dimension is not 16-byte aligned       */
    DLLM_ERR_UNSUPPORTED = -3, /* the current device is not sm_100                           */
    DLLM_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed                         */
    DLLM_ERR_ROW_RANGE = -5,   /* device-detected: a rows[] entry outside [0, M)               */
    DLLM_ERR_TIMEOUT = -6,     /* device-detected: a bounded wait inside a kernel ran out      */
    DLLM_ERR_WORKSPACE = -7,   /* workspace smaller than dllm_qgemm_workspace_bytes() asks     */
    DLLM_ERR_SCRATCH_LIMIT = -8, /* dllm_qgemm_noalloc: the call needs more scratch than the
                                    library's fixed array holds                              */
    DLLM_ERR_SCALE_RANGE = -9   /* device-detected: dllm_repack_q5k met a block scale d with
                                   |d| >= 4096, which the split form cannot hold (16 d is not a
                                   finite f16); those blocks' fifth-bit part is not usable      */
};

/* ------------------------------------------------------------------------------
 * Weights: load-time repack of GGUF blocks into the device tile layout.
 *
 * Input: row-major [N][K/256] GGUF blocks (144 bytes each for Q4_K, 210 for Q6_K),
 * on the device.  Output: the same bytes regrouped into tiles of 128 rows x 1
 * super-block, tile (t, s) at byte offset (t*(K/256) + s) * 128 * block_bytes, so
 * that one bulk copy brings a tile into shared memory.  Inside a tile:
 *   Q4_K (18432 B): quants [8][128 rows][16 B] | scale bytes [128][12] | d,dmin [128][2 x f16]
 *   Q6_K (26880 B): low bits [8][128][16 B] | high bits [4][128][16 B] |
 *                   int8 scales [128][16] | d [128][f16]
 * The repacked size equals the GGUF size (4.5 / 6.5625 bits per weight): nothing is
 * expanded (Architecture page, "Memory": the model stays resident once).
 * `gguf` and `dst` must not overlap.
 * ---------------------------------------------------------------------------- */
int dllm_repacked_bytes(dllm_qtype t, int64_t N, int64_t K, size_t* out_bytes); /* host pointer */
int dllm_repack_q4k(const void* gguf_blocks, int64_t N, int64_t K, void* dst, dllm_stream_t stream);
int dllm_repack_q6k(const void* gguf_blocks, int64_t N, int64_t K, void* dst, dllm_stream_t stream);
/* Q5_K: gguf_blocks is [N][K/256] 176-byte blocks; dst receives the Q4_K tile layout of
 * the split form, [N/128][2K/256] tiles of 18432 bytes (super-block s of a row at tile
 * column s for its low nibbles and K/256 + s for its fifth bits).  dllm_repacked_bytes
 * gives the size.  dllm_qgemm / dllm_qkv_qgemm / dllm_qgemm_noalloc take t = DLLM_Q5_K
 * with the ordinary K-wide activations.  A block scale with |d| >= 4096 (or not finite)
 * sets DLLM_ERR_SCALE_RANGE in the device error word (dllm_get_device_status). */
int dllm_repack_q5k(const void* gguf_blocks, int64_t N, int64_t K, void* dst, dllm_stream_t stream);
/* Q8_0: gguf_blocks is [N][K/32] 34-byte blocks (f16 d, then 32 int8 q).  dst receives
 * the codes as int8 [N][K] (row-major, read by TMA with the 128-byte swizzle) followed by
 * the block scales as f16 [N/128][K/256][128 rows][8]: 272 bytes per 256 weights, the
 * GGUF size.  dllm_qgemm / dllm_qkv_qgemm (one launch per projection) /
 * dllm_qgemm_noalloc take t = DLLM_Q8_0; the workspace holds only gathered rows. */
int dllm_repack_q80(const void* gguf_blocks, int64_t N, int64_t K, void* dst, dllm_stream_t stream);

/* ------------------------------------------------------------------------------
 * Activations: int8 with one f32 scale per 256 elements, plus scaled per-32 sums
 * (Architecture page, "Source map", kernels/qgemm.mojo row; "A forward pass",
 * step 2: quantized once, reused by Q/K/V and by gate/up).
 *
 * Rounding (the page leaves it open; this is the reading the library implements):
 * amax over the 256-block; iscale = 127/amax and scale = amax/127, each one IEEE
 * f32 division; qa = round-half-even(x * iscale) (one f32 multiply), clamped to
 * [-127, 127]; a block with amax = 0 has scale 0 and qa 0.
 *
 * x: f32 [M][ldx] row-major (ldx >= K, ldx % 4 == 0).  Outputs, with Mp = M rounded
 * up to a multiple of 16 (rows M..Mp-1 are written as zeros):
 *   q     int8  [K/256][Mp/8][16][8][16]: super-block s, 8-row group g, 16-byte chunk c
 *                (k = 256 s + 16 c + j), row r of the group, byte j.  Each group of 8
 *                rows x 16 bytes is one 128-byte core matrix of the tensor-core B operand.
 *   scale f32   [K/256][Mp]
 *   sums  f32   [K/256][Mp/8][4][8][4]: for the 8 sub-blocks of 32 of super-block s,
 *                v_j = scale * t_j (t_j the sum of the sub-block's 32 qa values, one f32
 *                multiply), stored as v_j = hi_j + lo_j where hi_j is v_j with its low 13
 *                mantissa bits cleared and lo_j = v_j - hi_j (exact).  Per super-block and
 *                8-row group, 512 bytes: [hi j0-3 | hi j4-7 | lo j0-3 | lo j4-7], each a
 *                [8 rows][4 floats] block (the tensor-core operand order of the min term).
 * dllm_act_bytes() gives the three sizes for (M, K).
 * ---------------------------------------------------------------------------- */
int dllm_act_bytes(int64_t M, int64_t K, size_t* q_bytes, size_t* scale_bytes, size_t* sums_bytes);
int dllm_quantize_act(const float* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* scale,
                      uint8_t* sums, dllm_stream_t stream);

/* ------------------------------------------------------------------------------
 * Quantization fused with the step that produces its input (Architecture page,
 * "A forward pass", steps 2 and 4).  Each layer runs RMSNorm before the Q/K/V and the
 * gate/up projections, and the final hidden state is normalised before the output
 * projection.  The FFN applies SiLU between gate/up and down.  The normalised or gated
 * f32 value is quantized in registers and never stored.  q, scale and sums have
 * exactly the layouts, sizes (dllm_act_bytes) and zero padding rows of
 * dllm_quantize_act, and the GEMM entry points consume them unchanged.
 *
 * Arithmetic (the page names the steps without formulas; these are the readings the
 * library implements).  Each value is formed in fp64 with correctly rounded
 * operations and rounded to f32 once.  The f32 is then quantized exactly as in
 * dllm_quantize_act.
 *   RMSNorm: ss = sum over the row's K elements of x^2, r = 1 / sqrt(ss / K + eps),
 *            y = f32((x * r) * gamma[k]).  The fp64 sum has one fixed order for
 *            every row count and row list (per super-block: each lane's 8 squares
 *            in element order, then a butterfly over 32 lanes; then slot l = the
 *            super-blocks l, l + 32, ... in order, and a butterfly over 32 slots),
 *            so a row list gives the full canvas's rows bit for bit.  Another order
 *            (the oracle's) can move y by one f32 rounding only when the fp64 value
 *            lies within about K * 2^-53 (relative) of a rounding boundary.
 *   SwiGLU:  h = f32((g / (1 + exp(-g))) * u).  exp is CUDA's fp64 exp.
 *
 * dllm_rmsnorm_quantize: x f32 [M][ldx] (ldx >= K, ldx % 4 == 0, K <= 65536), gamma f32 [K],
 *   eps > 0 and finite (else DLLM_ERR_ARG; eps = 0 would make an all-zero row 0/0).
 *   rows == NULL (n_rows = 0): all M canvas rows; the output has M rows.
 *   rows != NULL: device int32 list of n_rows >= 1 canvas rows (any order, duplicates
 *   allowed); output row i is canvas row rows[i] and the output has n_rows rows
 *   (size it with dllm_act_bytes(n_rows, K)).  This is the final RMSNorm on the
 *   requested rows only (Architecture page, "A forward pass", step 4), and the FFN
 *   input of the last layer, where only the requested positions continue past attention
 *   (step 3).  An entry outside [0, M) zero-fills its output row and sets
 *   DLLM_ERR_ROW_RANGE in the device error word.
 *   One CTA per output row (rounded up to 16 CTAs): min(K/256, 32) warps up to 12
 *   rows per SM, else min(ceil(K/1024), 4) warps that hold up to four super-blocks
 *   each in registers.
 * dllm_swiglu_quantize: gate, up f32 [M][ld] each (ld >= K, ld % 4 == 0).  They may
 *   be two column ranges of one buffer, e.g. the out_q/out_k pair of dllm_qkv_qgemm
 *   run on the gate and up weights with ld = 2 * K and up = gate + K.
 * Inputs are only read; the caller owns every buffer.  Both launch with programmatic
 * dependent launch, like dllm_quantize_act.  Errors: DLLM_ERR_ARG (sizes, eps, null),
 * DLLM_ERR_ALIGN (a pointer not 16-byte aligned or a leading dimension not a multiple
 * of 4), DLLM_ERR_UNSUPPORTED, DLLM_ERR_CUDA.
 * ---------------------------------------------------------------------------- */
int dllm_rmsnorm_quantize(const float* x, int64_t M, int64_t K, int64_t ldx, const float* gamma, float eps,
                          const int32_t* rows, int64_t n_rows, int8_t* q, float* scale, uint8_t* sums,
                          dllm_stream_t stream);
int dllm_swiglu_quantize(const float* gate, const float* up, int64_t M, int64_t K, int64_t ld, int8_t* q,
                         float* scale, uint8_t* sums, dllm_stream_t stream);

/* ------------------------------------------------------------------------------
 * GEMM: out[i][n] for n in [0, N) of one repacked weight matrix `w` (from
 * dllm_repack_*), activations (q, scale, sums) of an M-row canvas from
 * dllm_quantize_act.
 *   rows == NULL : i = m over all M rows; out is [M][ldo].
 *   rows != NULL : device int32 list of n_rows canvas rows (1 <= n_rows <= 32,
 *                  duplicates allowed, any order); out row i is canvas row rows[i];
 *                  out is [n_rows][ldo].  An entry outside [0, M) zero-fills its
 *                  output row and sets DLLM_ERR_ROW_RANGE in the device error word.
 *                  (Architecture page, "A forward pass", step 4: the output projection
 *                  runs only on the requested rows.)
 * ldo >= N, ldo % 4 == 0.  Results are deterministic and do not depend on M or on the
 * row set: a gathered row equals the same row of the full-canvas result bit for bit.
 *
 * workspace: device scratch owned by the caller, at least dllm_qgemm_workspace_bytes()
 * bytes (that size may be 0, and then workspace may be NULL); otherwise the call
 * returns DLLM_ERR_WORKSPACE.  It holds the gathered rows and, when a tile's K range
 * is split over several CTAs, their partial sums and one arrival counter per tile and
 * token super-tile.  The counters are the only contents that carry over between calls:
 * they occupy a fixed prefix (the first 64 KiB, or 4 bytes per tile and super-tile when
 * a call needs more) that no call's partial sums or gathered rows overlap, so one
 * workspace can serve calls of different shapes, provided each of them needs at most
 * 64 KiB of counters (ceil(N/128) x ceil(M/128) <= 16384).  It must be zero-filled
 * before its first use.  Every call that completes leaves each counter at a multiple of
 * 16, which is all the next call needs; a call that ends in DLLM_ERR_TIMEOUT may not, so
 * zero the workspace again after one.  Calls that share a workspace must be ordered on
 * one stream.
 * For dllm_qkv_qgemm pass N = Nq + 2*Nkv (Nq + Nkv without wv) and n_rows = 0.
 * ---------------------------------------------------------------------------- */
int dllm_qgemm_workspace_bytes(dllm_qtype t, int64_t N, int64_t K, int64_t M, int64_t n_rows, size_t* bytes);
int dllm_qgemm(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
               const uint8_t* sums, int64_t M, const int32_t* rows, int64_t n_rows, float* out, int64_t ldo,
               void* workspace, size_t workspace_bytes, dllm_stream_t stream);

/* ------------------------------------------------------------------------------
 * dllm_qgemm with no caller workspace.  The paper has no counterpart of this entry
 * point; it is a convenience of this library.
 *
 * Same operation, arguments, results and device-detected errors as dllm_qgemm, but
 * the scratch (gathered rows, split-K partial sums, arrival counters) is a fixed
 * array of DLLM_NOALLOC_SCRATCH_BYTES bytes in the library's own device memory, one
 * per device, reserved when the library's device code is loaded on that device.  It
 * serves callers that cannot obtain device memory where they call: a host runtime
 * that passes this library only buffers it already owns and has no allocator to
 * lend it; a step where a cudaMalloc, which may synchronize the whole device, would
 * stall work on other streams; plain C code that would rather not size, own and
 * zero a workspace.
 *
 *   - Limit: a call whose scratch need (dllm_qgemm_workspace_bytes() for the same
 *     arguments) exceeds DLLM_NOALLOC_SCRATCH_BYTES returns DLLM_ERR_SCRATCH_LIMIT
 *     and launches nothing.  32 MiB holds every single projection of LLaDA-8B and
 *     Dream-7B on canvases of up to 384 rows (the largest, Dream-7B's down
 *     projection at 384 rows, needs 26.25 MiB) and the output projection on up to
 *     32 rows.
 *   - Zero state: only the arrival counters must start at zero.  The call clears
 *     the counters it uses on `stream` (an asynchronous memset of at most a few KB)
 *     before its kernel runs, so nothing carries over between calls, including from
 *     a call that ended in DLLM_ERR_TIMEOUT.  The partial sums and gathered rows are
 *     written in full before they are read.
 *   - Set-up: the first call on a device, with that device current, looks up the
 *     array's device address (cudaGetSymbolAddress, which also loads the library's
 *     device code there) and sets the kernel's shared-memory limit; later calls on
 *     that device reuse both.  Make that first call before any stream capture begins.
 *   - Races: all calls on a device share its one array.  Calls that overlap in time
 *     (issued to different streams, or from host threads without ordering between
 *     their streams) race on it and give wrong results; issue every call of this
 *     entry point on a device to one stream.
 * ---------------------------------------------------------------------------- */
#define DLLM_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int dllm_qgemm_noalloc(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
                       const uint8_t* sums, int64_t M, const int32_t* rows, int64_t n_rows, float* out,
                       int64_t ldo, dllm_stream_t stream);

/* ------------------------------------------------------------------------------
 * Several projections of one quantized activation in one launch (Architecture page,
 * "A forward pass", step 2: quantize once, reuse for Q, K and V; the same holds for
 * the FFN's gate and up).  wq has Nq rows, wk and wv Nkv rows; wv == NULL runs two
 * projections (e.g. gate and up).  oq is [M][ldo_q], ok and ov are [M][ldo_kv].
 * ---------------------------------------------------------------------------- */
int dllm_qkv_qgemm(const void* wq, const void* wk, const void* wv, dllm_qtype t, int64_t Nq, int64_t Nkv,
                   int64_t K, const int8_t* q, const float* scale, const uint8_t* sums, int64_t M, float* oq,
                   int64_t ldo_q, float* ok, float* ov, int64_t ldo_kv, void* workspace, size_t workspace_bytes,
                   dllm_stream_t stream);

/* ------------------------------------------------------------------------------
 * Attention: bidirectional (no mask) softmax attention over the canvas, the step
 * between the Q/K/V and the output projections (Architecture page, "A forward
 * pass", step 2: attention runs over all L positions with no mask; heatdrop card,
 * "Key highlights": f16 tensor cores with an online softmax).
 *
 *   o[i][h][:] = sum_j softmax_j( q[i][h] . k[j][g] / sqrt(dh) ) v[j][g][:],
 *   g = h / (H / Hkv)   (grouped-query attention when Hkv < H)
 *
 * q: f16 [Lq][H][dh]; k, v: f16 [Lk][Hkv][dh] (contiguous, 16-byte aligned; q and k
 * as they come out of RoPE); o: f32 [Lq][H][dh], written, may not overlap the inputs.
 * dh must be 128 (LLaDA-8B and Dream-7B).  Lq == 0 is a no-op; Lk must be >= 1.
 * Arithmetic: Q K^T on f16 tensor cores with f32 accumulation; the softmax in f32
 * with base-2 exponents and a running maximum raised only when a block maximum
 * exceeds it by more than 2^8; the weights rounded to f16 for P V on the tensor
 * cores (f32 accumulation), the normaliser summed in f32 before that rounding, so each
 * normalised weight is off by at most about 2^-11 of itself plus the f32 effects.
 * One CTA per (128 queries, head) while that grid fits one wave of CTAs on the
 * device's SMs, else one CTA per (256 queries, head) with the two query tiles in
 * ping-pong (dllm_debug_attention_tiles gives the choice); programmatic dependent
 * launch like the GEMM.
 * Errors: DLLM_ERR_ARG (sizes, dh != 128, H % Hkv, null), DLLM_ERR_ALIGN,
 * DLLM_ERR_UNSUPPORTED, DLLM_ERR_CUDA; DLLM_ERR_TIMEOUT in the device error word.
 * ---------------------------------------------------------------------------- */
int dllm_attention(const void* q, const void* k, const void* v, int64_t Lq, int64_t Lk, int64_t H, int64_t Hkv,
                   int64_t dh, float* o, dllm_stream_t stream);

/* Synchronizes `stream`, then returns and clears the device error word
 * (DLLM_OK, DLLM_ERR_ROW_RANGE or DLLM_ERR_TIMEOUT). */
int dllm_get_device_status(dllm_stream_t stream);
const char* dllm_status_string(int code);

/* ------------------------------------------------------------------------------
 * Test and measurement entry points (not on the hot path).
 * ---------------------------------------------------------------------------- */

/* Per-sub-block integer dot products on CUDA cores, for bit-exact checking:
 * dots[m][n][j] (int32, [M][N][K/32] for Q4_K with q in 0..15, [M][N][K/16] for
 * Q6_K with q - 32), from the repacked weights and the quantized activations. */
int dllm_debug_subblock_dots(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, int64_t M,
                             int32_t* dots, dllm_stream_t stream);

/* The per-super-block integers the int8 tensor-core path forms, read back from
 * tensor memory instead of being combined: S[m][n][s] = sum_j sc_j * dot_j (Q4_K) or
 * sum_j sc_j * dot_j with q - 32 (Q6_K), int32 [M][N][K/256].  Same kernel and
 * schedule as dllm_qgemm with the f32 epilogue replaced. */
int dllm_debug_sb_ints(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
                       const uint8_t* sums, int64_t M, int32_t* S, dllm_stream_t stream);

/* Bounded-wait check: launches one CTA of the GEMM kernel whose producer issues no
 * copy, so the first barrier wait of every other role runs out (after about 2 s).
 * The kernel then records DLLM_ERR_TIMEOUT in the device error word, frees its tensor
 * memory and returns; the context stays usable.  Returns the launch status; read the
 * device status with dllm_get_device_status(). */
int dllm_debug_bounded_wait(dllm_stream_t stream);

/* The same check for the attention kernels: one CTA of the one-tile kernel (two_tiles ==
 * 0) or of the two-tile kernel (two_tiles != 0) whose TMA producers issue no copy, so
 * every other role's first wait runs out (after about 2 s).  The kernel records
 * DLLM_ERR_TIMEOUT in the device error word, frees its tensor memory and returns without
 * storing anything; its tensor maps cover the library's own scratch array.  Returns the
 * launch status. */
int dllm_debug_attention_stall(int two_tiles, dllm_stream_t stream);

/* The work split the GEMM would use for a weight of n_tiles 128-row tiles, K inputs,
 * an M-row canvas (n_rows requested rows, 0 for all) on a device with `sms` SMs.
 * Host only: no device is touched.  out (host, 8 entries) receives kc (K-chunks per
 * tile of the uniform split), full_tiles, tail_k and tail_big (the tail split: tiles
 * [0, full_tiles) whole, the first tail_big of the rest in tail_k + 1 K-pieces, the
 * others in tail_k; tail_k = 0 means the uniform split), n_units, n_st (token
 * super-tiles), mu (tokens per super-tile) and the workspace bytes.  The pages have no
 * counterpart; the split is this library's scheduling.  DLLM_ERR_ARG on bad sizes. */
int dllm_debug_plan(int64_t n_tiles, int64_t K, int64_t M, int64_t n_rows, int sms, int64_t* out);

/* Query tiles of 128 rows per CTA that dllm_attention uses for Lq queries and H heads
 * on a device with `sms` SMs: 1 while ceil(Lq / 128) * H <= sms (one wave of one-tile
 * CTAs), else 2.  Host only.  DLLM_ERR_ARG when an argument is below 1. */
int dllm_debug_attention_tiles(int64_t Lq, int64_t H, int sms);

/* int8 tensor-core throughput probe: on each of `ctas` CTAs, `issuers` warps (1..4)
 * each issue `iters` back-to-back tcgen05 kind::i8 MMAs of 128 x n x 32 into their own
 * n_acc accumulators, with A in tensor memory (a_from_tmem != 0) or shared memory.
 * Writes elapsed device nanoseconds per CTA to ns_out (device, [ctas] uint64).
 * 16 <= n <= 256, n % 16 == 0, n * n_acc * issuers <= 448, iters % 8 == 0. */
int dllm_bench_mma_i8(int n, int n_acc, int a_from_tmem, int issuers, int iters, int ctas,
                      unsigned long long* ns_out, dllm_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DLLM_QGEMM_H */
