/*
 * hq.h -- C ABI of the HyperQuant tile codec for NVIDIA B200 (sm_100a).
 *
 * The codec is the data-parallel path of "HyperQuant: A Rate-Distortion-Optimal Quantization
 * Pipeline for Large Language and Diffusion Models" (Domb, Sackstein, Solberg; summarised on
 * gist.science, Technical Summary, "Methodology: The HyperQuant Pipeline"):
 *   step 1  per-tile Randomized Hadamard Transform  RHT_n(x) = H_n D x,
 *   step 2  nearest-point quantization to the E8, D4, A2 or Z lattice (integer embedding),
 *   step 3  lossless bit-stripping and per-tile Rice coding of the lattice indices,
 *   step 4  subtractive dither U ~ Uniform(V(Lambda)) on the KV path, so inner products stay
 *           unbiased per vector.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument named as a device pointer must point to memory of the current CUDA
 *     device; the library never allocates or frees memory and keeps no state between calls
 *     besides cached driver entry points and the fixed scratch array of hq_encode_noalloc; it
 *     never synchronises except in hq_status_read.  All work is enqueued on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and the call returns at once.
 *   - The synchronous return value reports argument errors (HQ_ERR_ARG, HQ_ERR_UNSUPPORTED) and
 *     launch failures (HQ_ERR_CUDA).  Errors found by the kernels (non-finite input, too small
 *     an output, a corrupt stream, a bounded wait that ran out) are written to a status word in
 *     the caller's workspace `ws` and read with hq_status_read.
 *   - The workspace is caller-owned device memory of at least hq_workspace_bytes(...) bytes,
 *     256-byte aligned.  Calls that share a workspace must not overlap on the GPU.
 *   - Tiles.  A weight W[rows, cols] is row-major; tile (r, jt) is W[r, jt*n : (jt+1)*n], along
 *     the input-channel axis.  Tile index t = jt*rows + r.  Chunk (jt, rb) holds the tiles of
 *     rows [32 rb, min(32 rb + 32, rows)) of tile column jt; chunk index c = jt*RB + rb with
 *     RB = ceil(rows / 32).  Each chunk starts on a 32-bit word; chunk_word[c] is its word
 *     offset in `bits`, chunk_word[C] the total number of words.
 *   - A KV tensor [B, H, S, D] (contiguous) is coded as rows = B*H*S, cols = n = D: one tile per
 *     head vector, the random signs shared by every head and token (per-layer seed), the dither
 *     fresh per (b, h, s) and group of four coefficients.
 *   - Dither (Methodology step 4, "Subtractive Dither"): U uniform on the Voronoi cell of the
 *     lattice, in its quantizer's coordinates (u for Z, D4, E8; (P, Q) = (2 u0, u1 2/sqrt3) for
 *     A2).  Group g of four consecutive coefficients of a tile draws one Philox4x32-10 block, key
 *     = seed, counter (c_lo, c1, 0x80000000 | g, c_hi): c = s, c1 = b*H + h for KV row (b, h, s);
 *     c = row, c1 = tile column for dithered weights.  r_i = box (w_i >> 8) 2^-24 with box 1 (Z)
 *     or 2, and U = r - Q(r) per lattice block (E8 blocks take groups 2b, 2b+1).
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HQ_FORMAT_VERSION 2

/* Lattices of Methodology step 2. */
typedef enum { HQ_Z = 0, HQ_A2 = 1, HQ_D4 = 2, HQ_E8 = 3 } hq_lattice_t;

/* Element types of the dense side (input of encode, output of decode). */
typedef enum { HQ_BF16 = 0, HQ_F32 = 1 } hq_dtype_t;

typedef enum {
    HQ_OK = 0,
    HQ_ERR_ARG = 1,          /* bad argument (null pointer, size, alignment, range)          */
    HQ_ERR_UNSUPPORTED = 2,  /* valid but not provided (e.g. fp32 input with n = 256)       */
    HQ_ERR_CAPACITY = 3,     /* device: `bits` too small; detail = words needed              */
    HQ_ERR_NONFINITE = 4,    /* device: a tile held NaN/Inf (coded as zeros); detail = count */
    HQ_ERR_CORRUPT = 5,      /* device: stream inconsistent with meta / chunk_word            */
    HQ_ERR_TIMEOUT = 6,      /* device: a bounded wait on another block ran out               */
    HQ_ERR_RANGE = 7,        /* value outside a representable range                          */
    HQ_ERR_CUDA = 8          /* a CUDA runtime call failed                                    */
} hq_status_t;

/*
 * Codec parameters.
 *   tile    n in {64, 128, 256}, the RHT tile length (Methodology step 1, "e.g. 128").
 *   lattice one of hq_lattice_t (Methodology step 2).
 *   step    beta > 0: lattice units per normalised coefficient.  A tile with RMS s is coded as
 *           u = H_n D x / (sqrt(n) * bf16(s) * beta).  Allowed range [2^-8, 2^6]; the range
 *           keeps every code below 2^15 in magnitude and every Rice parameter below 10.
 *           0 selects hq_step_for_rate(lattice, tile, bps).
 *   bps     target payload bits per scalar, used only when step == 0.
 *   seed    64-bit seed of the sign diagonal D (and of the KV dither).
 */
typedef struct {
    int32_t tile;
    int32_t lattice;
    float step;
    float bps;
    uint64_t seed;
} hq_params_t;

/*
 * An encoded tensor.  The caller owns the four device arrays and the struct; encode fills them
 * and the scalar fields, decode reads them.
 *   rows, cols  dense shape (KV: rows = B*H*S, cols = D)
 *   kv_S        S of the KV layout (dither counter); 0 for weights
 *   p           parameters with the step resolved (never 0 after encode)
 *   kv          0 plain; 1 KV rows with the dither; 2 weights with the dither (hq_encode_dither);
 *               3 KV rows with the dither and the dense rotation (hq_kv_encode_dense)
 *   version     HQ_FORMAT_VERSION
 *   scale       [T] bf16 bit patterns of the per-tile RMS (0 = all-zero tile)
 *   meta        [T] k | (sum q << 4): the tile's Rice parameter and unary total
 *   chunk_word  [C + 1] word offset of each chunk, [C] = total words
 *   bits        [cap_words] the bitstream; cap_words >= hq_encode_bound_words(...) always
 *               suffices, a smaller buffer yields HQ_ERR_CAPACITY with the needed size
 *   kv_s0       KV: the position of the code's first token in every sequence (0 unless the
 *               tokens were appended with hq_kv_encode_at)
 */
typedef struct {
    int64_t rows, cols;
    int64_t kv_S;
    hq_params_t p;
    int32_t kv;
    int32_t version;
    uint16_t* scale;
    uint16_t* meta;
    uint32_t* chunk_word;
    uint32_t* bits;
    int64_t cap_words;
    int64_t kv_s0;
} hq_code_t;

/* Number of tiles T and chunks C of a rows x cols tensor with tile length n; -1 if invalid. */
int64_t hq_num_tiles(int64_t rows, int64_t cols, int32_t tile);
int64_t hq_num_chunks(int64_t rows, int64_t cols, int32_t tile);

/* Worst-case bitstream words for any finite input (a multiple of 4); -1 if invalid. */
int64_t hq_encode_bound_words(int64_t rows, int64_t cols, const hq_params_t* p);

/* Workspace bytes needed by any call on a rows x cols tensor with these parameters. */
size_t hq_workspace_bytes(int64_t rows, int64_t cols, const hq_params_t* p);

/*
 * Step for a target payload rate from the high-resolution approximation of an entropy-coded
 * lattice quantizer on Gaussian coefficients (the RHT output is close to Gaussian, Methodology
 * step 1): beta = 2^(h - R) / V^(1/d) with h = log2(sqrt(2 pi e)) and V, d the cell volume
 * and dimension of the lattice.  A starting point; hq_encode_count gives the realised rate for
 * an exact search (the method lands the realised rate about 0.01 bps from its target,
 * Methodology step 3).
 */
float hq_step_for_rate(int32_t lattice, int32_t tile, float bps);

/*
 * Encode a weight (Methodology steps 1-3).
 *   x      device, [rows, cols] row-major, dtype elements, 16-byte aligned base, cols % tile == 0
 *   out    host struct: scale/meta/chunk_word/bits/cap_words set by the caller, the rest filled
 *   ws     device workspace (hq_workspace_bytes), ws_bytes its size
 * Device errors: HQ_ERR_NONFINITE (tile coded as zeros), HQ_ERR_CAPACITY, HQ_ERR_TIMEOUT.
 */
hq_status_t hq_encode(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                      hq_code_t* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Several weights in one launch: the same codes, chunk offsets and bitstreams as one hq_encode per
 * item, with the tiles of all items taken by one persistent grid, so that one tensor's last wave
 * runs beside the next tensor's tiles instead of leaving SMs idle.
 *   count  1 .. HQ_BATCH_MAX items; all share p.tile, p.lattice and dtype (HQ_ERR_UNSUPPORTED
 *          otherwise); each item its own x, shape, step, seed and out (as for hq_encode)
 *   ws     device workspace of at least hq_encode_batch_workspace_bytes(count, items) bytes (one
 *          header and every item's look-back states); the status word reports the whole batch
 * Returns HQ_ERR_ARG for an invalid item; nothing is launched then.
 */
#define HQ_BATCH_MAX 16
typedef struct {
    const void* x;     /* device, [rows, cols] row-major, dtype elements, 16-byte aligned        */
    hq_dtype_t dtype;  /* HQ_BF16 or HQ_F32                                                     */
    int64_t rows, cols;
    hq_params_t p;
    hq_code_t* out;    /* host struct as for hq_encode: arrays set by the caller, the rest filled */
} hq_encode_item_t;
size_t hq_encode_batch_workspace_bytes(int32_t count, const hq_encode_item_t* items);
hq_status_t hq_encode_batch(int32_t count, const hq_encode_item_t* items, void* ws, size_t ws_bytes, void* stream);

/*
 * Several KV tensors (or token appends) in one launch, e.g. the keys and values of every layer for
 * one decoding step: the same codes as one hq_kv_encode_at (hq_kv_encode when s0 = 0) per item.
 * Each item: kv[B, H, S, D] (device, contiguous, 16-byte aligned), the positions s0 .. s0 + S - 1,
 * its own step and seed.  All items share D = p.tile = 128, p.lattice and dtype
 * (HQ_ERR_UNSUPPORTED otherwise).  ws: hq_kv_encode_batch_workspace_bytes(count, items) bytes.
 */
typedef struct {
    const void* kv;
    hq_dtype_t dtype;
    int64_t B, H, S, D, s0;
    hq_params_t p;
    hq_code_t* out;
} hq_kv_item_t;
size_t hq_kv_encode_batch_workspace_bytes(int32_t count, const hq_kv_item_t* items);
hq_status_t hq_kv_encode_batch(int32_t count, const hq_kv_item_t* items, void* ws, size_t ws_bytes, void* stream);

/*
 * Weight-path dither option: as hq_encode, with the dither of tile (row, tile column) added
 * before quantization (the method applies the dither to the KV cache; here any lattice, any
 * shape).  out->kv = 2; hq_decode takes the dither off again.
 */
hq_status_t hq_encode_dither(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                             hq_code_t* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Decode a weight: y[rows, cols] (device, dtype, 16-byte aligned) = D H_n p * (bf16(s) beta /
 * sqrt(n)) per tile, p the lattice point (minus the dither for codes with kv = 2); bf16 output
 * is the binary32 value rounded to nearest even.  Device errors: HQ_ERR_CORRUPT (tile written
 * as zeros).
 */
hq_status_t hq_decode(const hq_code_t* code, void* y, hq_dtype_t dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Several weight codes in one launch: the same output as one hq_decode per item, the tiles of all
 * items taken by one grid.  count 1 .. HQ_BATCH_MAX; all codes share p.tile and p.lattice, are
 * weight codes without dither (kv = 0), and all outputs one dtype (HQ_ERR_UNSUPPORTED
 * otherwise).  ws: at least 64 bytes; the status word reports the whole batch.
 */
typedef struct {
    const hq_code_t* code;
    void* y;           /* device, [rows, cols], dtype elements, 16-byte aligned */
    hq_dtype_t dtype;  /* HQ_BF16 or HQ_F32                                     */
} hq_decode_item_t;
hq_status_t hq_decode_batch(int32_t count, const hq_decode_item_t* items, void* ws, size_t ws_bytes, void* stream);

/*
 * Encode a KV tensor kv[B, H, S, D] (device, contiguous) with D == p->tile and the dither
 * (Methodology step 4): the dither U of each head vector, uniform on the Voronoi cell of
 * p->lattice (any of the four; the method's choice is D4), is added before quantization.
 */
hq_status_t hq_kv_encode(const void* kv, hq_dtype_t dtype, int64_t B, int64_t H, int64_t S, int64_t D,
                         const hq_params_t* p, hq_code_t* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Token append: encode kv[B, H, S, D] as the tokens s0 .. s0 + S - 1 of every (b, h) sequence, so
 * the dither of token (b, h, s0 + s) is the one a whole-sequence encode would draw (for a decode
 * step, S = 1: one head vector per (b, h)).  Each tile is coded on its own, so the tiles equal
 * those of the whole-sequence code; the chunks (32 consecutive rows) follow this call's rows.
 * out->kv_s0 = s0 >= 0.
 */
hq_status_t hq_kv_encode_at(const void* kv, hq_dtype_t dtype, int64_t B, int64_t H, int64_t S, int64_t D, int64_t s0,
                            const hq_params_t* p, hq_code_t* out, void* ws, size_t ws_bytes, void* stream);

/* Decode a KV tensor: the dither is regenerated and subtracted before the inverse transform. */
hq_status_t hq_kv_decode(const hq_code_t* code, void* kv, hq_dtype_t dtype, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * Dense-rotation KV variant (Methodology step 4, "Bias Correction for KV Cache": the per-layer
 * rotation may be a dense Haar-random orthogonal matrix instead of the sign diagonal).  Each head
 * vector x of kv[B, H, S, D] (device, contiguous, D == p->tile == 128) is coded as
 *   u = (Q x) / (bf16(s) beta),  s the RMS of x (the codec's scale, zero and non-finite vectors as
 *   in hq_encode),
 * then quantized with the KV dither of token (b, h, s0 + s), bit-stripped and Rice-coded exactly
 * like hq_kv_encode_at: one tile per head vector, chunks of 32 rows.  u_j is the binary32 fma chain
 * over i = 0 .. 127 of Q[j][i] x_i from 0, multiplied by the binary32 1 / (bf16(s) beta).
 *   Q    fp32 [128, 128] row-major (device, 4-byte aligned), orthogonal; the caller draws it (from
 *        the Haar measure for the method's variant) and passes the same Q to the decode.  No sign
 *        diagonal and no 1/sqrt(n) factor are applied: Q is the whole rotation.
 *   ws   at least hq_kv_dense_workspace_bytes(B*H*S) bytes (holds the coefficients between the
 *        rotation and the codec).
 * out->kv = 3, out->kv_s0 = s0.  D other than 128: HQ_ERR_UNSUPPORTED.  Device errors as
 * hq_kv_encode_at (HQ_ERR_NONFINITE counts the non-finite head vectors).
 */
size_t hq_kv_dense_workspace_bytes(int64_t rows);
hq_status_t hq_kv_encode_dense(const void* kv, hq_dtype_t dtype, int64_t B, int64_t H, int64_t S, int64_t D,
                               int64_t s0, const float* Q, const hq_params_t* p, hq_code_t* out, void* ws,
                               size_t ws_bytes, void* stream);

/*
 * Decode a dense-rotation KV code (code->kv == 3) into kv[rows, 128] (device, bf16 or fp32,
 * 16-byte aligned): p = lattice point minus the dither in u units, x_hat = (Q^T p) (bf16(s) beta)
 * in binary32 (fma over j = 0 .. 127, then one product), rounded to nearest even for bf16.
 * ws: hq_kv_dense_workspace_bytes(rows).  Device errors: HQ_ERR_CORRUPT (tile decoded as zeros).
 */
hq_status_t hq_kv_decode_dense(const hq_code_t* code, const float* Q, void* kv, hq_dtype_t dtype, void* ws,
                               size_t ws_bytes, void* stream);

/*
 * Lattice quantization, bit-stripping and Rice coding of caller-given normalised coefficients
 * (Methodology steps 2-3, and step 4's dither when kv != 0): u[tiles, tile] fp32 device array in
 * lattice units, one tile per row, chunks of 32 consecutive rows.  v_out (device, optional,
 * int32 [tiles, tile]) receives the integer codes: Z and D4 the point itself, E8 twice the point,
 * A2 (P, Q) with the point at (P/2, Q sqrt(3)/2).  kv = 1: row t is token (t / kv_S, t % kv_S)
 * (kv_S <= 0: one head); kv = 2: row t is the weight tile (t, 0).
 * out->scale may be NULL.  This entry point checks codes and bitstreams bit for bit.
 */
hq_status_t hq_quantize_coeffs(const float* u, int64_t tiles, const hq_params_t* p, int32_t kv, int64_t kv_S,
                               int32_t* v_out, hq_code_t* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Count-only encode: writes the total payload bits of encoding x (no bitstream) to
 * *bits_out (device uint64).  Used to search the step for an exact rate.
 */
hq_status_t hq_encode_count(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                            int32_t kv, int64_t kv_S, uint64_t* bits_out, void* ws, size_t ws_bytes, void* stream);

/*
 * The weight's integer lattice codes, for an int8 tensor-core GEMM in the RHT domain: v_out
 * [rows, cols] int8 (device, 16-byte aligned) holds the codes of tile (r, jt) at columns jt n ..
 * (E8: twice the lattice point; Z, D4: the point), g_out [cols / n, rows] fp32 (device) the tile's
 * scale ((s_hat beta) c_n) c_L with c_L = 1/2 for E8, 1 otherwise, in binary32, so that the tile
 * decodes to D H_n (v g).  Tiles with a code outside [-127, 127] are written as zeros and
 * reported as HQ_ERR_RANGE; tiles of a corrupt stream as zeros with HQ_ERR_CORRUPT.
 * Supported: Z, D4, E8 codes without dither, n = 128 or 256 (HQ_ERR_UNSUPPORTED otherwise).
 */
hq_status_t hq_decode_int8(const hq_code_t* code, int8_t* v_out, float* g_out, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * Grouped int8 GEMM on the tensor cores (the method's int8 MMA path on the post-RHT lattice
 * codes; abstract and "Experimental Results"):
 *   Y[m, r] = sa[m] * sum_t g[t, r] S(m, r, t),  S(m, r, t) = sum_{j = 128 t}^{128 t + 127} A[m, j] V[r, j]
 * A int8 [M, K] (activations after the same RHT, D H_n per tile of 128), sa fp32 [M], V int8
 * [N, K] and g fp32 [K / 128, N] as written by hq_decode_int8, Y fp32 [M, N]; all device,
 * row-major, 16-byte aligned.  The group sums are exact; the scales are applied in binary32 as
 * acc = fma(S, g, acc) over t = 0, 1, ... from acc = 0, then Y = acc * sa[m].  group must be 128;
 * M and N multiples of 128, K a multiple of 128 up to 2^20 (HQ_ERR_UNSUPPORTED / HQ_ERR_ARG
 * otherwise).  ws: at least 64 bytes; a bounded wait that ran out reports HQ_ERR_TIMEOUT there.
 * The CTA tile is 128 rows by 128, 64 or 32 columns (the widest whose tiles occupy every SM); the
 * result does not depend on it.
 */
hq_status_t hq_gemm_int8(const int8_t* A, const float* sa, int64_t M, const int8_t* V, const float* g, int64_t N,
                         int64_t K, int32_t group, float* Y, void* ws, size_t ws_bytes, void* stream);

/*
 * The same product as hq_decode_int8 followed by hq_gemm_int8, with the decode fused into the
 * GEMM: producer warps decode the weight's code (Rice codes, unstrip) straight into the tensor
 * cores' int8 operand stages, so the int8 codes never reach global memory.  W = the code's
 * weight [N, K] (N = code->rows, K = code->cols, a multiple of 128 each; n = 128; Z, D4 or E8
 * without dither, HQ_ERR_UNSUPPORTED otherwise); A int8 [M, K] row-major (M >= 1; rows past M of
 * the last 128-row tile are zeros), sa fp32 [M], Y fp32 [M, N]; all device, 16-byte aligned.
 *   Y[m, r] = sa[m] * sum_t g[t, r] S(m, r, t)
 * bit for bit as the two-call path: exact int32 group sums, acc = fma(S, g, acc) over t = 0, 1, ...
 * from 0 in binary32, then Y = acc * sa[m]; tiles with a code outside int8 are zero (HQ_ERR_RANGE),
 * corrupt tiles too (HQ_ERR_CORRUPT).  A CTA takes 128 activation rows against a slab of 32
 * weight rows (one chunk of the code per K group) over all K groups, so every output element's
 * chain stays in one CTA (two 128-row activation tiles per slab once M > 128).  Products with
 * (M / 256) (N / 32) (K / 128) of 2^31 or more: HQ_ERR_UNSUPPORTED.  ws: at least
 * hq_gemm_code_workspace_bytes(M, N, K) bytes (the status word); calls sharing ws must not overlap.
 */
size_t hq_gemm_code_workspace_bytes(int64_t M, int64_t N, int64_t K);
hq_status_t hq_gemm_code(const int8_t* A, const float* sa, int64_t M, const hq_code_t* code, float* Y, void* ws,
                         size_t ws_bytes, void* stream);

/* Result of a step search, written to device memory. */
typedef struct {
    float step;            /* the chosen step beta                                          */
    int32_t probes;        /* count-only passes made                                        */
    uint64_t payload_bits; /* payload bits of encoding x at `step` (Methodology step 3 rate) */
} hq_rate_result_t;

/*
 * Exact-rate mode: search the step whose payload rate is p->bps (in [1, 8]) on this tensor, the
 * per-tensor counterpart of the method's claim that the realised rate lands about 0.01 bps from
 * any target (Methodology step 3, Rice coding).  Up to `max_probes` (1 .. 64; 0 means 16)
 * count-only encodes, each followed by a one-thread update on the device: the first probe is
 * p->step if it is > 0, else hq_step_for_rate; while only one side of the target has been seen
 * the next probe is a Newton step in log2(step) with slope -1 bit per scalar per doubling; once
 * the target is bracketed, regula falsi on the binary32 bit patterns of the step, with a
 * bisection whenever the same side moves twice in a row.  The search stops at the first probe
 * within tol_bps of the target (tol_bps <= 0 means 0.005; at most 1), when the bracket closes to
 * adjacent binary32 steps, at the
 * ends of the step range [2^-8, 64], or after max_probes passes; `result` (device) then holds
 * the probe closest to the target.  Everything runs on `stream` without a host synchronisation
 * (a CUDA graph may capture it).  ws: at least hq_workspace_bytes(rows, cols, p) bytes.
 * Errors: HQ_ERR_ARG for invalid arguments, as hq_encode_count; device errors in ws.
 */
hq_status_t hq_step_search(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                           int32_t kv, int64_t kv_S, int32_t max_probes, float tol_bps, hq_rate_result_t* result,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronise `stream`, then read the status word of `ws`: returns HQ_OK or the most severe
 * device error (TIMEOUT, CORRUPT, CAPACITY, NONFINITE in that order) and, if detail is not NULL,
 * its detail value (capacity: words needed; non-finite: tiles affected).
 */
hq_status_t hq_status_read(const void* ws, void* stream, int64_t* detail);

/* Static description of a status code. */
const char* hq_status_str(hq_status_t s);

/* HQ_FORMAT_VERSION of the built library. */
int32_t hq_version(void);

/*
 * Allocation-free weight encode.  The method has no counterpart for this entry point; it exists
 * for callers that must not allocate GPU memory at encode time -- an inference engine that
 * owns its memory pool and forbids further allocations while it serves, code running between
 * two synchronisation points where cudaMalloc / cudaFree would stall every stream of the
 * device, or a host language runtime without a device allocator.  Such a caller passes only the
 * input and the output arrays (out->scale, meta, chunk_word, bits as for hq_encode).
 *
 * The encoder's scratch (status word, work counter, one look-back slot per block of 128 tiles)
 * is a fixed array of HQ_NOALLOC_SCRATCH_BYTES compiled into the library, present on every GPU
 * that loads it until the process exits.  It covers tensors with
 *     64 + 8 * (cols / tile) * ceil(rows / (tile == 256 ? 64 : 128)) <= HQ_NOALLOC_SCRATCH_BYTES
 * (e.g. 8192 x 28672 at tile 256, 16384 x 8192 at tile 128); larger tensors get HQ_ERR_RANGE
 * and nothing is enqueued.  Like the other entry points it makes the device that holds x (device
 * or managed memory) the calling thread's current device.  The first call on a device looks the
 * array's device address up (cudaGetSymbolAddress) for that device, and so does the first call
 * after that device's primary context was replaced (cudaDeviceReset destroys the array's
 * contents and may move it); make such a call before capturing the stream into a graph.  All
 * calls share the one array and each call clears it on `stream` before its kernel runs, so calls
 * whose work overlaps on the GPU (different streams without ordering) race and must not be
 * issued.  Device errors (capacity, non-finite input, timeout) are copied
 * as the status bit word (1 << hq_status_t) to *status_out (device uint32) when it is not
 * NULL.  No allocation, no synchronisation.
 */
#define HQ_NOALLOC_SCRATCH_BYTES (128 * 1024)
hq_status_t hq_encode_noalloc(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                              hq_code_t* out, uint32_t* status_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
