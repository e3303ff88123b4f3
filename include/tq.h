/*
 * tq.h -- C ABI of libtq: TurboQuant-style KV-cache compression on NVIDIA B200 (sm_100a).
 *
 * The hot path, and the page that defines each step:
 *   - key encode:   norm separation, seeded Haar rotation, nearest Lloyd-Max level, bit packing
 *                   ("KV Cache API", compressors.py MSECompressor.compress; "aitherkvcache",
 *                   TurboQuant.encode returning uint8 codes plus f32 norms);
 *   - value encode: grouped affine min/max quantization with fp16 scale and zero
 *                   ("KV Cache API", values.py quantize_values);
 *   - decode:       unpack, codebook gather, inverse rotation, norm rescale; affine dequant for values
 *                   (compressors.py MSECompressor.decompress; values.py dequantize_values);
 *   - decode-step attention scored directly against the packed keys
 *                   ("KV Cache API", store.py TurboQuantKVCache.attention_scores / attend;
 *                   "turbo-attn", the split-K paged decode kernel with a fused query rotation).
 *
 * Conventions shared by every entry point
 *   - Every call returns a tq_status.  On anything but TQ_OK, tq_last_error() returns a message (owned by
 *     the library, valid until the next call on the same thread) that names the offending argument.
 *   - Device pointers are caller-owned (allocate them with any allocator, e.g. PyTorch).  No entry point
 *     allocates or frees device memory except tq_codec_create / tq_codec_destroy.
 *   - Kernels are enqueued on the caller's stream (a cudaStream_t passed as void*; NULL = the legacy
 *     default stream) and return without synchronising.  Outputs are fully overwritten.
 *   - Argument errors are detected on the host before anything is enqueued; nothing is launched then.
 *   - Preconditions that are NOT checked on the device: inputs are finite (no NaN/Inf), pointers
 *     reference allocations of the stated sizes, and outputs do not overlap inputs.
 *   - Half-precision data are IEEE binary16 passed as void* / uint16_t*.
 *   - Supported head dims for the device kernels: 64, 128, 256.  Key bits 1..4.  Value bits 2, 3, 4, 8
 *     with group 32 or group == head_dim (the page's "token" scale layout).
 *   - Packed rows are LSB-first bitstreams: index j of a row occupies bits [j*b, (j+1)*b) of the row read
 *     as little-endian bytes; a row has (d*b + 7) / 8 bytes and rows are contiguous.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tq_status {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,   /* null pointer, negative count, misaligned pointer or stride, bad layout */
    TQ_ERR_UNSUPPORTED = 2,   /* a head_dim / bits / group / GQA combination the kernels do not implement */
    TQ_ERR_CUDA = 3,          /* a CUDA runtime call failed; the message carries cudaGetErrorString */
    TQ_ERR_DEVICE_FLAG = 4    /* a kernel's bounded wait expired and it raised the device error flag */
} tq_status;

typedef enum tq_dtype {
    TQ_F16 = 0,               /* IEEE binary16 */
    TQ_F32 = 1                /* IEEE binary32 */
} tq_dtype;

/* Message for the last non-TQ_OK status returned on this thread ("" if none). */
const char* tq_last_error(void);

/* ABI version of this header (major * 100 + minor). */
int tq_version(void);

/* --------------------------------------------------------------------------------------------------
 * Host parameter builders (CPU only; no device needed).
 * ------------------------------------------------------------------------------------------------ */

/*
 * tq_make_rotation -- the seeded Haar rotation Pi ("KV Cache API", compressors.py MSECompressor.__init__:
 * G = randn(d, d); Q, R = qr(G); Pi = Q * sign(diag R), zero signs taken as +1; "TurboQuant: A KV Cache
 * Compression Technique", step 1, Haar-distributed orthogonal matrix).
 *   d        head dimension, 2..1024.
 *   seed     G[i][j] is standard normal draw i*d + j of SplitMix64(seed) through Box-Muller (pairs of
 *            consecutive outputs u1, u2: r = sqrt(-2 ln u1'), draws r cos(2 pi u2'), r sin(2 pi u2'), with
 *            u1' = (u1 >> 11 + 0.5) 2^-53 and u2' = (u2 >> 11) 2^-53).
 *   pi       out, nullable: d*d doubles, row-major; the rotated vector is y = Pi x.
 *   pi_f16   out, nullable: d*d binary16, the nearest fp16 of each entry (Pi_op, what the kernels use).
 * Errors: TQ_ERR_INVALID_ARG for d out of range or both outputs NULL.
 */
tq_status tq_make_rotation(int d, uint64_t seed, double* pi, uint16_t* pi_f16);

/* Rotation kinds of tq_make_rotation_ex / tq_codec_create_ex. */
typedef enum tq_rotation {
    TQ_ROT_HAAR = 0,          /* the seeded Haar rotation of tq_make_rotation */
    TQ_ROT_HADAMARD = 1       /* the seeded randomized Walsh-Hadamard rotation below */
} tq_rotation;

/*
 * tq_make_rotation_ex -- tq_make_rotation for either rotation kind.  TQ_ROT_HADAMARD ("turbo-attn", The
 * codec, "Hadamard rotation": a Walsh-Hadamard transform spreads outlier channels across the vector and the
 * queries are rotated the same way) is Pi = H diag(s) / sqrt(d): H the Sylvester Hadamard matrix
 * (H[i][j] = (-1)^popcount(i & j)), s_j = -1 if the top bit of SplitMix64(seed) output j (0-based) is set,
 * else +1.  The page fixes neither the signs nor the scale; these make Pi orthogonal and the rotated
 * coordinates of an isotropic vector follow the same marginal, so the same codebook applies.
 *   rotation  TQ_ROT_HAAR or TQ_ROT_HADAMARD (then d must be a power of two).
 * Errors: TQ_ERR_INVALID_ARG for a bad kind, d out of range or not a power of two (Hadamard), or both
 * outputs NULL.
 */
tq_status tq_make_rotation_ex(int d, uint64_t seed, int rotation, double* pi, uint16_t* pi_f16);

/*
 * tq_build_codebook -- data-independent Lloyd-Max levels for one rotated coordinate ("KV Cache API",
 * compressors.py calls _solve_codebook(head_dim, bits), body not shown; "TurboQuant: A KV Cache
 * Compression Technique", step 2, optimal codebooks from a mathematical derivation).  The coordinate
 * density is the exact marginal of a uniform point on the unit sphere S^(d-1):
 * f(x) proportional to (1 - x^2)^((d-3)/2) on [-1, 1].
 *   d, bits       2 <= d <= 65536, 1 <= bits <= 8.
 *   centroids     out, nullable: 2^bits doubles, ascending (c*).
 *   centroids_f16 out, nullable: 2^bits binary16, the nearest fp16 of each level (c_op).
 *   boundaries    out, nullable: 2^bits - 1 floats, midpoints of adjacent c_op levels (exact in fp32).
 *   distortion    out, nullable: D = E ||y - Q(y)||^2 for a uniform unit vector y quantized coordinate-wise
 *                 with c_op and these boundaries.
 * Errors: TQ_ERR_INVALID_ARG for d or bits out of range.
 */
tq_status tq_build_codebook(int d, int bits, double* centroids, uint16_t* centroids_f16,
                            float* boundaries, double* distortion);

/* --------------------------------------------------------------------------------------------------
 * Key codec handle: Pi_op, Pi_op^T, c_op, boundaries and search tables resident on the current device.
 * ------------------------------------------------------------------------------------------------ */

typedef struct tq_codec tq_codec;

/*
 * tq_codec_create -- build the rotation and codebook for (d, k_bits, seed) on the host and upload them to
 * the current CUDA device (synchronously, with cudaMalloc/cudaMemcpy; not a hot-path call).
 *   d      64, 128 or 256.       k_bits 1..4.
 *   out    receives the handle; the handle belongs to the device that was current at creation.
 * Errors: TQ_ERR_UNSUPPORTED for other d / bits, TQ_ERR_CUDA if the device allocation fails.
 */
tq_status tq_codec_create(int d, int k_bits, uint64_t seed, tq_codec** out);

/*
 * tq_codec_create_ex -- tq_codec_create with the rotation kind (tq_rotation).  Every kernel is the same:
 * the rotation is a d x d fp16 matrix multiplied on the tensor cores whichever kind it is.
 * Errors: as tq_codec_create, plus TQ_ERR_INVALID_ARG for an unknown kind.
 */
tq_status tq_codec_create_ex(int d, int k_bits, uint64_t seed, int rotation, tq_codec** out);

/* The rotation kind a codec was created with (TQ_ROT_HAAR for tq_codec_create). */
tq_status tq_codec_rotation(const tq_codec* codec, int* rotation);

/* Free a codec (NULL is accepted).  The caller must ensure no enqueued work still uses it. */
tq_status tq_codec_destroy(tq_codec* codec);

/* Read back a codec's parameters (any out pointer may be NULL). */
tq_status tq_codec_info(const tq_codec* codec, int* d, int* k_bits, uint64_t* seed);

/*
 * tq_encode_k -- key encode ("KV Cache API", compressors.py MSECompressor.compress: norms, normalise,
 * rotate, nearest centroid, pack; "aitherkvcache": fp16 [..., 128] -> uint8 [..., 64] at 4 bits + f32 norms).
 *   x             in, device, binary16 rows: row r starts at x + r * x_row_stride (elements).  x must be
 *                 16-byte aligned and x_row_stride a multiple of 8 with x_row_stride >= d.
 *   n             number of rows (0 is a no-op).
 *   slot_mapping  in, device, nullable, int64[n]: destination row of each input row in the output arrays
 *                 (a paged pool); a negative entry skips the row.  NULL: row r goes to row r.
 *   packed        out, device: rows of d*k_bits/8 bytes.      norms  out, device: float per row.
 * Per row: n = ||x||_2 (fp32); y = Pi_op x / (n + 1e-8); index j = #{i : t_i < y_j}; LSB-first packing.
 * Indices agree with the fp64 definition except where y_j lies within ~1e-6 of a boundary t_i.
 */
tq_status tq_encode_k(const tq_codec* codec, const void* x, int64_t n, int64_t x_row_stride,
                      const int64_t* slot_mapping, uint8_t* packed, float* norms, void* stream);

/*
 * tq_decode_k -- key decode ("KV Cache API", compressors.py MSECompressor.decompress: centroids[idx] @ Pi,
 * times the norm).
 *   packed, norms in, device: n rows as written by tq_encode_k (contiguous).
 *   out           out, device: n rows of d elements of out_dtype (TQ_F16 or TQ_F32), 16-byte aligned.
 * x_hat = n * Pi_op^T c_op[idx], accumulated in fp32 on the tensor cores.
 */
tq_status tq_decode_k(const tq_codec* codec, const uint8_t* packed, const float* norms, int64_t n,
                      void* out, int out_dtype, void* stream);

/* --------------------------------------------------------------------------------------------------
 * Value codec (no handle: the format is fully described by d, bits and group).
 * ------------------------------------------------------------------------------------------------ */

/*
 * tq_encode_v -- grouped affine value quantizer ("KV Cache API", values.py quantize_values).
 *   d, bits, group  d in {64,128,256}; bits in {2,3,4,8}; group 32 or d (the page's "token" layout).
 *   x               in, device, binary16 rows with stride x_row_stride (elements; 16-byte aligned rows).
 *   slot_mapping    as for tq_encode_k.
 *   data            out, device: rows of (d*bits+7)/8 bytes.
 *   scales, zeros   out, device: binary16 [rows][d/group].
 * Per group, in IEEE fp32 with one rounding per operation and in this order:
 *   scale = max((max - min) / (2^bits - 1), 1e-12); zero = min;
 *   q = clamp(round_half_even((x - zero) / scale), 0, 2^bits - 1);
 * scale and zero are then stored as fp16 (round to nearest even).  The result is bit-exact with that
 * definition.
 */
tq_status tq_encode_v(int d, int bits, int group, const void* x, int64_t n, int64_t x_row_stride,
                      const int64_t* slot_mapping, uint8_t* data, void* scales, void* zeros, void* stream);

/*
 * tq_decode_v -- value dequantization ("KV Cache API", values.py dequantize_values):
 * x_hat = float(q) * float(scale16) + float(zero16), two fp32 operations, then stored as out_dtype
 * (TQ_F32 exact; TQ_F16 round to nearest even).  Inputs are contiguous rows as tq_encode_v writes them.
 */
tq_status tq_decode_v(int d, int bits, int group, const uint8_t* data, const void* scales,
                      const void* zeros, int64_t n, void* out, int out_dtype, void* stream);

/* --------------------------------------------------------------------------------------------------
 * Decode-step attention over the compressed cache.
 * ------------------------------------------------------------------------------------------------ */

/*
 * Cache layouts.  Every pool array (K payload, K norms, V data, V scales, V zeros) is indexed by a row:
 *   contiguous: row = (b * num_kv_heads + h) * max_seq_len + t;
 *   paged:      row = (block_table[b * max_blocks + t / block_size] * num_kv_heads + h) * block_size
 *                     + t % block_size.
 * Sequence b attends to tokens 0 .. seq_lens[b]-1 (all max_seq_len tokens if seq_lens is NULL in the
 * contiguous layout; seq_lens is required for the paged layout).  The kernels clamp seq_lens[b] to
 * [0, max_seq_len] in the contiguous layout and to [0, max_blocks * block_size] in the paged one, so a length
 * past the cache attends to the whole addressable sequence and never reads beyond its rows or its
 * block-table row.  Every block_table entry below the (clamped) length must name a block of the pools.  Query head hq reads kv head
 * hq / (num_q_heads / num_kv_heads).
 */
typedef struct tq_attend_args {
    int batch;                 /* B >= 1 */
    int num_q_heads;           /* H_q, a multiple of num_kv_heads; H_q / H_kv <= 8 */
    int num_kv_heads;          /* H_kv >= 1 */
    int head_dim;              /* must equal the codec's d */
    int v_bits;                /* 2, 3, 4 or 8 */
    int v_group;               /* 32 or head_dim */
    float scale;               /* softmax scale; 0 means 1/sqrt(head_dim) ("KV Cache API", attention_scores) */
    int64_t max_seq_len;       /* contiguous layout: T per (b, h); paged: ignored */
    const int32_t* block_table;/* NULL: contiguous layout.  Else device int32 [batch][max_blocks] */
    int max_blocks;            /* paged: columns of block_table */
    int block_size;            /* paged: tokens per block (16) */
    const int32_t* seq_lens;   /* device int32 [batch], nullable in the contiguous layout */
    const void* q;             /* device binary16 [batch][num_q_heads][head_dim] */
    const uint8_t* k_packed;   /* device pool of key rows (tq_encode_k format) */
    const float* k_norms;      /* device pool of key norms */
    const uint8_t* v_data;     /* device pool of value rows (tq_encode_v format) */
    const void* v_scales;      /* device binary16 pool [rows][head_dim / v_group] */
    const void* v_zeros;       /* device binary16 pool [rows][head_dim / v_group] */
    float* out;                /* device float [batch][num_q_heads][head_dim] */
    void* workspace;           /* device scratch (16-byte aligned) of at least the size
                                  tq_attend_workspace_bytes reports: the prepared query fragments of each
                                  (sequence, kv head), then the split-K partials.  Its contents need no
                                  initialisation and are overwritten by every call. */
    size_t workspace_bytes;
} tq_attend_args;

/*
 * tq_attend_workspace_bytes -- bytes of workspace tq_attend_decode needs for these arguments on the current
 * device: (head_dim / 16 * 32 + 2) * 16 bytes per (sequence, kv head) for the prepared query, plus the split-K
 * partials when the sequence axis is split.  Only the shape fields of args are read.  The size assumes the
 * most splits any key width can use (four attention CTAs per SM); a launch whose kernel keeps fewer CTAs
 * resident splits less and uses a prefix of the same workspace.
 * Errors: the same argument checks as tq_attend_decode (TQ_ERR_INVALID_ARG / TQ_ERR_UNSUPPORTED).
 */
tq_status tq_attend_workspace_bytes(const tq_attend_args* args, size_t* bytes);

/*
 * tq_attend_decode -- one decode step of attention against the compressed cache ("KV Cache API",
 * store.py attention_scores + softmax + attend; "turbo-attn", split-K paged decode with the query
 * rotated once).  For each (b, hq) with h = hq / G:
 *   q_rot = Pi_op q;  s_t = scale * n_t * <q_rot, c_op[idx_t]>;  p = softmax(s);
 *   out = sum_t p_t * (q_t * scale16_t + zero16_t)   (the value dequantized inside the kernel).
 * No fp16 key or value is written to memory.  A sequence of length 0 yields zeros.  A small first kernel
 * rotates and splits the query once per (sequence, kv head); the attention kernel is its programmatic
 * dependent on the same stream.  When the sequence axis is split over several CTAs, a third kernel (again a
 * programmatic dependent) merges the per-split partials with a log-sum-exp rescale.  Calls that overlap on
 * the GPU must use distinct workspaces.
 */
tq_status tq_attend_decode(const tq_codec* codec, const tq_attend_args* args, void* stream);

/*
 * tq_attend_scores -- the attention logits of the compressed path, for score-fidelity measurements
 * ("turboquant-pytorch", V3: Attention Score Accuracy -- cosine similarity and top-1 / top-5 matches of the
 * scores against the uncompressed ones): s[b][hq][t] = scale * n_t * <Pi_op q, c_op[idx_t]> in fp32, the
 * same scores tq_attend_decode softmaxes.
 *   scores  out, device float [batch][num_q_heads][L], L = max_seq_len (contiguous) or max_blocks * 16
 *           (paged); positions at or past a sequence's length are -inf.
 * args->out and the value pool are not used; args->workspace needs at least tq_attend_workspace_bytes bytes
 * (only its prepared-query part is written).
 * Errors: as tq_attend_decode.
 */
tq_status tq_attend_scores(const tq_codec* codec, const tq_attend_args* args, float* scores, void* stream);

/* --------------------------------------------------------------------------------------------------
 * Attention with a window of recent uncompressed tokens.
 * ------------------------------------------------------------------------------------------------ */

/* Largest window per (sequence, kv head) tq_attend_decode_window accepts. */
#define TQ_ATTEND_WINDOW_MAX 256

typedef struct tq_attend_window {
    const void* k;             /* device binary16 [batch][num_kv_heads][max_len][head_dim]: recent keys as stored */
    const void* v;             /* device binary16, same layout: recent values as stored */
    const int32_t* lens;       /* device int32 [batch]: window tokens of each sequence (clamped to 0..max_len);
                                  NULL: max_len for every sequence */
    int max_len;               /* 1..TQ_ATTEND_WINDOW_MAX */
} tq_attend_window;

/*
 * tq_attend_window_workspace_bytes -- workspace bytes tq_attend_decode_window needs (as
 * tq_attend_workspace_bytes, with one more partial per (sequence, kv head) for the window).
 */
tq_status tq_attend_window_workspace_bytes(const tq_attend_args* args, const tq_attend_window* window,
                                           size_t* bytes);

/*
 * tq_attend_decode_window -- tq_attend_decode over the compressed cache plus a window of recent tokens kept
 * uncompressed ("KV Cache API", store.py TurboQuantKVCache: attention_scores concatenates the quantized
 * part's scores with scale * query @ key_buffer^T; the softmax runs over both; attend adds the quantized
 * part's weights times the dequantized values and the buffer's weights times the buffer's values).  The
 * window's scores are fp32 dot products of the fp16 query and keys, times the same scale; one extra CTA per
 * (sequence, kv head) computes them and its partial (max, sum, weighted values) enters the same split merge.
 * A sequence whose compressed part and window are both empty yields zeros.
 * Errors: as tq_attend_decode, plus TQ_ERR_INVALID_ARG for a NULL window, NULL k or v, max_len outside
 * 1..TQ_ATTEND_WINDOW_MAX or misaligned (16-byte) k / v.
 */
tq_status tq_attend_decode_window(const tq_codec* codec, const tq_attend_args* args, const tq_attend_window* window,
                                  void* stream);

/*
 * TQ_ATTEND_SCRATCH_BYTES -- size of the library-owned scratch used by tq_attend_decode_noalloc (4 MiB).
 * That array lives in the library's device image, so every GPU that loads libtq holds it until the process
 * exits, whether or not the entry point is ever called.
 */
#define TQ_ATTEND_SCRATCH_BYTES (4u << 20)

/*
 * tq_attend_decode_noalloc -- the same decode-step attention as tq_attend_decode, for callers that cannot
 * allocate device memory at all: code running inside a CUDA graph that is being captured or replayed, a
 * serving loop whose memory pool is fixed once at start-up, or a host process that only receives a
 * stream and buffers from elsewhere.  The pages have no counterpart; this is a property of this library.
 *
 * Instead of a caller workspace it uses a fixed scratch array of TQ_ATTEND_SCRATCH_BYTES that the library
 * declares at file scope in device memory; args->workspace and args->workspace_bytes are ignored.  The
 * entry point calls no allocator (no cudaMalloc, no cudaFree, nothing that allocates).
 *   - Set-up: the first call on each device looks up the scratch array's device address with
 *     cudaGetSymbolAddress (with that device current) and caches it for the life of the process; make that
 *     first call outside any stream capture.  The cached address belongs to the device's primary context:
 *     after cudaDeviceReset (or any reset of that context) it is stale, so do not call this entry point
 *     again in a process that has reset the device.
 *   - Limit: the check uses the size tq_attend_workspace_bytes reports for the same arguments (planned for
 *     the most splits any key width can use); when that exceeds TQ_ATTEND_SCRATCH_BYTES the call is
 *     rejected with TQ_ERR_INVALID_ARG and a message giving both sizes, even if this codec's key width
 *     would launch fewer splits.  Use tq_attend_decode with a caller workspace for such shapes.
 *   - Sharing: all calls on a device share the one array and it keeps the last call's contents; nothing
 *     in it needs to start at zero, since every launch overwrites the part it reads.  Calls that can
 *     overlap on the GPU (different streams without ordering, or different threads) race on it and must
 *     be serialised by the caller.
 * Errors: as tq_attend_decode, plus TQ_ERR_CUDA if the address lookup fails.
 */
tq_status tq_attend_decode_noalloc(const tq_codec* codec, const tq_attend_args* args, void* stream);

/* --------------------------------------------------------------------------------------------------
 * QJL residual keys.
 * ------------------------------------------------------------------------------------------------ */

/*
 * tq_codec_create_qjl -- a key codec for QJL residual keys ("KV Cache API", compressors.py
 * TurboQuantCompressorV2: the MSE compressor at bits - 1, then one sign bit per row of a seeded Gaussian matrix S
 * applied to the residual r of the MSE reconstruction, and ||r||).
 *   bits      total bits per coordinate, 2..5; the MSE stage uses bits - 1 (tq_codec_info reports bits - 1, so
 *             the codec also serves tq_encode_k / tq_decode_k / tq_attend_decode as an ordinary key codec).
 *   S         d x d, entry (i, j) = Gaussian draw i * d + j of this library's generator (SplitMix64 and
 *             Box-Muller) seeded with seed + 10000; the tensor cores multiply by S_op = fp16(S).
 * Errors: as tq_codec_create_ex, TQ_ERR_UNSUPPORTED for bits outside 2..5.
 */
tq_status tq_codec_create_qjl(int d, int bits, uint64_t seed, int rotation, tq_codec** out);

/*
 * tq_make_qjl_matrix -- the sketch S of a QJL codec with this d and seed, on the host (row-major d*d): entry
 * (i, j) is Gaussian draw i * d + j of the generator seeded with seed + 10000; s_f16 (nullable) receives
 * fp16(S), the operand the kernels use.  Either output may be NULL, not both.
 */
tq_status tq_make_qjl_matrix(int d, uint64_t seed, double* s, uint16_t* s_f16);

/* tq_codec_qjl_bits -- the total bits of a QJL codec; 0 for a codec made by tq_codec_create / _ex. */
tq_status tq_codec_qjl_bits(const tq_codec* codec, int* bits);

/*
 * tq_encode_k_qjl -- QJL key encode ("KV Cache API", compressors.py TurboQuantCompressorV2.compress):
 *   the MSE stage, exactly tq_encode_k with this codec at bits - 1, into packed and norms; then
 *   k_mse = n * Pi_op^T c_op[idx];  r = x - k_mse (f32);  rho = ||r|| (f32);  sign_i = ((S_op r)_i >= 0).
 *   signs     out, device: rows of d/8 bytes; coordinate i is bit i of the row's LSB-first bitstream, 1 for +1.
 *   rho       out, device: float per row.
 * Rows, strides, alignment and the slot mapping (which places packed, norms, signs and rho alike) are those of
 * tq_encode_k.  k_mse multiplies fp16 codebook values by fp16 Pi_op and S_op r multiplies r, split into fp16
 * hi + lo halves, by fp16 S_op, both with f32 accumulation: a sign can differ from an exact evaluation only
 * where (S_op r)_i lies within about 1e-6 * ||S_op row i|| * ||x|| of zero.  Launches two kernels on `stream`.
 * Errors: as tq_encode_k; TQ_ERR_INVALID_ARG for a codec not made by tq_codec_create_qjl or NULL signs / rho.
 */
tq_status tq_encode_k_qjl(const tq_codec* codec, const void* x, int64_t n, int64_t x_row_stride,
                          const int64_t* slot_mapping, uint8_t* packed, float* norms, uint8_t* signs, float* rho,
                          void* stream);

/* QJL key pools beside the MSE-stage pools of tq_attend_args, indexed by the same rows. */
typedef struct tq_qjl_keys {
    const uint8_t* signs;      /* device pool of sign rows (tq_encode_k_qjl format: d/8 bytes per row) */
    const float* rho;          /* device pool of residual norms */
} tq_qjl_keys;

/*
 * tq_attend_qjl_workspace_bytes -- workspace bytes tq_attend_decode_qjl needs: as tq_attend_workspace_bytes, with
 * a second block of prepared query fragments (the sketched query) per (sequence, kv head).
 */
tq_status tq_attend_qjl_workspace_bytes(const tq_attend_args* args, size_t* bytes);

/*
 * tq_attend_decode_qjl -- decode attention over QJL residual keys ("KV Cache API", store.py attention_scores
 * with compressors.py asymmetric_attention_scores): for each (b, hq), kv head h = hq / G,
 *   s_t = scale * ( n_t <Pi_op q, c_op[idx_t]> + rho_t sqrt(pi/2) / d <S_op q, sign_t> ),  sign_t in {-1, +1}^d,
 *   p = softmax(s);  out = sum_t p_t * (q_t * scale16_t + zero16_t),
 * i.e. tq_attend_decode with the estimator's second term in every logit.  args describes the MSE-stage pools
 * (the codec's bits - 1 codes and norms) and the values exactly as for tq_attend_decode; keys adds the sign and
 * rho pools.  The prepared query now has two halves (Pi_op q and S_op q, each fp16 hi + lo fragments); the sign
 * pairs enter the tensor cores as fp16 +-1.  Values: 2 or 4 bits in groups of 32.
 * Errors: as tq_attend_decode; TQ_ERR_INVALID_ARG for a codec not made by tq_codec_create_qjl, NULL or
 * misaligned (16-byte) signs / rho; TQ_ERR_UNSUPPORTED for another value format.
 */
tq_status tq_attend_decode_qjl(const tq_codec* codec, const tq_attend_args* args, const tq_qjl_keys* keys,
                               void* stream);

/* --------------------------------------------------------------------------------------------------
 * Diagnostics.
 * ------------------------------------------------------------------------------------------------ */

/*
 * Read (and optionally clear) the current device's error flag, which a kernel sets when one of its bounded
 * waits expires.  Synchronises the device.  flag_out receives 0 when nothing was raised.
 */
tq_status tq_read_device_flag(int* flag_out, int clear);

/*
 * tq_stream_status -- wait for the work queued on `stream` (that stream only; other streams keep running) and
 * report whether any kernel's bounded wait has expired: TQ_ERR_DEVICE_FLAG (with the flag in tq_last_error)
 * if the device's error flag is set, else TQ_OK.  clear != 0 resets the flag after reading it.  A kernel
 * whose wait expired has stopped its roles, let every copy and tensor-core operation it issued complete,
 * released its tensor memory and returned, so the context stays usable; its outputs are incomplete.
 */
tq_status tq_stream_status(void* stream, int clear);

/*
 * tq_debug_encode_k_stalled -- a test of the bounded-wait path: tq_encode_k on n contiguous rows (row stride d)
 * with the first 128-row tile's copy withheld in every CTA and every wait limited to wait_limit_cycles
 * (1000 .. 2^31).  Nothing waits on a copy or an MMA that was issued and is still in flight: the waits on
 * the withheld tile run out, the kernel raises the device flag, drains what it issued, frees its tensor memory
 * and returns.  Follow with tq_stream_status to read the result.  The outputs are not meaningful.
 */
tq_status tq_debug_encode_k_stalled(const tq_codec* codec, const void* x, int64_t n, uint8_t* packed, float* norms,
                                    long long wait_limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
