// libtq: the C ABI of include/tq.h over the sm_100a kernels.  Host-side validation, codec lifecycle,
// TMA descriptor creation and template dispatch live here; the kernels are in the included headers.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "tq_attend_kernel.cuh"
#include "tq_qjl_kernel.cuh"
#include "tq_codec_kernels.cuh"
#include "tq_internal.h"

using namespace tq;
using namespace tq::dev;

// ------------------------------------------------------------------------------------------ helpers

namespace {

#define TQ_CUDA(call, what)                                                                        \
    do {                                                                                           \
        cudaError_t e_ = (call);                                                                   \
        if (e_ != cudaSuccess) return fail(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_));    \
    } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = v > 0 ? v : 148;
    }
    return cache[dev];
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D fp16 tensor map over rows x cols (row stride in elements), 128B swizzle, box of 64 cols x box_rows.
tq_status make_tmap_f16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride,
                        uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_stride * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return TQ_OK;
}

// 2-D tensor map for the decoded keys: rows x cols of fp16 or fp32 (dense rows), 64B swizzle, box of
// 64 bytes x 32 rows (one warp's patch).
tq_status make_tmap_out(CUtensorMap* map, void* base, uint64_t rows, uint64_t cols, bool f32) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    const uint64_t elt = f32 ? 4 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * elt};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(64 / elt), 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return TQ_OK;
}

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename K>
cudaError_t allow_smem(K kernel, uint32_t bytes, std::atomic<uint64_t>& done_mask) {
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (done_mask.load() & bit) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e == cudaSuccess) done_mask.fetch_or(bit);
    return e;
}

bool supported_d(int d) { return d == 64 || d == 128 || d == 256; }

}  // namespace

// ------------------------------------------------------------------------------------------- codec

struct tq_codec {
    int d = 0, bits = 0, device = 0, rotation = TQ_ROT_HAAR;
    uint64_t seed = 0;
    __half* pi_op = nullptr;        // d x d, rotated = Pi_op x
    __half* pi_op_t = nullptr;      // Pi_op^T, the decode-side B operand
    uint32_t* enc_lut = nullptr;    // kGridCells grid cells: boundary bits | count below (low 4 bits)
    uint32_t* pair_lut = nullptr;   // 2^(2 bits) half2 pairs
    CUtensorMap tmap_pi, tmap_pit;
    int qjl_bits = 0;               // QJL codec: total bits per coordinate (bits + 1), else 0
    __half* s_op = nullptr;         // QJL codec: the d x d Gaussian sketch S_op = fp16(S), row-major
    float s_row_max = 0.f;          // QJL codec: max over rows of ||S_op row||
};

namespace {

// Grid table of the encode search (see encode_k_kernel): cell c holds the y whose u = 64 y + 128, rounded to a
// multiple of 2^-7, has integer part c, so the 256 cells cover y in [-2, 2) (|y| <= ||Pi_op|| < 1.01).  Each
// cell is taken as the closed range u in [c - 1/128, c + 1], wider than the values that can reach it: a
// boundary below it is below every y in the cell, and one inside it is decided by y > B.  Entry = bits of the
// one boundary inside the cell (+inf if none) OR the count of boundaries below the cell; the boundaries,
// midpoints of fp16 levels, have at least 4 zero low bits in fp32 (checked), and no cell holds two of them for
// any supported d and bits (checked: the closest pair, d = 256 at 4 bits, is 0.016 apart, above the widened
// cell's 0.01575).
tq_status build_grid_lut(int bits, const float* t, std::vector<uint32_t>& lut) {
    const int nb = (1 << bits) - 1;
    lut.assign(kGridCells, 0);
    for (int c = 0; c < kGridCells; ++c) {
        const double lo = (c - kGridOffset - 1.0 / 128) / kGridRes, hi = (c + 1.0 - kGridOffset) / kGridRes;
        uint32_t below = 0;
        int inside = 0;
        float b = INFINITY;
        for (int i = 0; i < nb; ++i) {
            const double ti = t[i];
            if (ti < lo) ++below;
            else if (ti <= hi) { ++inside; b = t[i]; }
        }
        if (inside > 1) return fail(TQ_ERR_UNSUPPORTED, "codebook boundaries closer than the search grid (bits=%d)", bits);
        uint32_t bb;
        std::memcpy(&bb, &b, 4);
        if (bb & 15u) return fail(TQ_ERR_UNSUPPORTED, "a codebook boundary needs more than 28 significant bits");
        lut[c] = bb | below;
    }
    return TQ_OK;
}

// Grid of the encode search for 5..8 bits (see encode_k_kernel): cell(y) = bits 5..14 of
// fma(sat(fma(y, s, 0.5)), 1023.75, 1.5 * 2^18) with s = 0.499 / max|t|, a monotone map of y onto 1024 cells
// that the device computes with the same two fp32 FMAs.  Every boundary must land in a cell of its own; then for
// y in cell c the boundaries of lower cells are below y, those of higher cells above it, and the one in c (if
// any) is decided by y > B.  Entry c = {bits of the boundary in c (+inf if none), boundaries in lower cells},
// stored kWideCopies times side by side (copy r of entry c at 8-byte slot kWideCopies c + r, so lanes reading
// different copies of nearby entries use different banks); the word after the entries holds s.
uint32_t wide_cell(float y, float s) {
    float u = std::fmaf(y, s, 0.5f);
    u = (u > 0.f) ? ((u < 1.f) ? u : 1.f) : 0.f;               // saturate; NaN -> 0
    const float g = std::fmaf(u, 1023.75f, 393216.0f);            // 1.5 * 2^18, ulp 2^-5: the cell at bits 5..14
    uint32_t b;
    std::memcpy(&b, &g, 4);
    return (b >> 5) & (kWideCells - 1);
}

tq_status build_wide_grid(int bits, const float* t, std::vector<uint32_t>& lut) {
    const int nb = (1 << bits) - 1;
    float tmax = 0.f;
    for (int i = 0; i < nb; ++i) tmax = std::fmax(tmax, std::fabs(t[i]));
    const float s = static_cast<float>(0.499 / tmax);
    std::vector<uint32_t> bnd(kWideCells), cnt(kWideCells);
    const float inf = INFINITY;
    uint32_t inf_bits;
    std::memcpy(&inf_bits, &inf, 4);
    for (int c = 0; c < kWideCells; ++c) bnd[c] = inf_bits;
    int prev = -1;
    for (int i = 0; i < nb; ++i) {
        const int c = static_cast<int>(wide_cell(t[i], s));
        if (c <= prev) return fail(TQ_ERR_UNSUPPORTED, "codebook boundaries closer than the wide search grid (bits=%d)", bits);
        std::memcpy(&bnd[c], &t[i], 4);
        prev = c;
    }
    for (int c = 0, below = 0, i = 0; c < kWideCells; ++c) {
        while (i < nb && static_cast<int>(wide_cell(t[i], s)) < c) { ++i; ++below; }
        cnt[c] = static_cast<uint32_t>(below);
    }
    lut.assign(2 * kWideCells * kWideCopies + 4, 0);
    for (int c = 0; c < kWideCells; ++c)
        for (int r = 0; r < kWideCopies; ++r) {
            lut[2 * (kWideCopies * c + r)] = bnd[c];
            lut[2 * (kWideCopies * c + r) + 1] = cnt[c];
        }
    std::memcpy(&lut[2 * kWideCells * kWideCopies], &s, 4);
    return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_codec_create_ex(int d, int k_bits, uint64_t seed, int rotation, tq_codec** out) {
    clear_error();
    if (!out) return fail(TQ_ERR_INVALID_ARG, "tq_codec_create: out is NULL");
    *out = nullptr;
    if (!supported_d(d)) return fail(TQ_ERR_UNSUPPORTED, "tq_codec_create: d=%d (supported: 64, 128, 256)", d);
    if (k_bits < 1 || k_bits > 8) return fail(TQ_ERR_UNSUPPORTED, "tq_codec_create: k_bits=%d (supported: 1..8)", k_bits);
    if (k_bits > 4 && d > 128)
        return fail(TQ_ERR_UNSUPPORTED,
                    "tq_codec_create: k_bits=%d needs d <= 128 (at d=256 the key decoder's shared memory holds no wider "
                    "rows)", k_bits);
    if (rotation != TQ_ROT_HAAR && rotation != TQ_ROT_HADAMARD)
        return fail(TQ_ERR_INVALID_ARG, "tq_codec_create: rotation=%d (TQ_ROT_HAAR or TQ_ROT_HADAMARD)", rotation);
    const size_t dd = static_cast<size_t>(d) * d;
    std::vector<uint16_t> pi16(dd), pit16(dd);
    std::vector<double> pi(dd);
    host_rotation_of(rotation, d, seed, pi.data());
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) {
            pi16[static_cast<size_t>(i) * d + j] = f64_to_f16(pi[static_cast<size_t>(i) * d + j]);
            pit16[static_cast<size_t>(j) * d + i] = pi16[static_cast<size_t>(i) * d + j];
        }
    const int k = 1 << k_bits;
    std::vector<uint16_t> c16(k);
    std::vector<float> t(k - 1);
    tq_status st = tq_build_codebook(d, k_bits, nullptr, c16.data(), t.data(), nullptr);
    if (st != TQ_OK) return st;
    std::vector<uint32_t> lut;
    std::vector<uint32_t> pairs;
    if (k_bits <= 4) {
        // search grid and code-pair table (a pair of codes -> half2 of levels, the first code in the low half)
        if ((st = build_grid_lut(k_bits, t.data(), lut)) != TQ_OK) return st;
        pairs.resize(1u << (2 * k_bits));
        for (uint32_t key = 0; key < pairs.size(); ++key)
            pairs[key] = static_cast<uint32_t>(c16[key & (k - 1)]) | (static_cast<uint32_t>(c16[key >> k_bits]) << 16);
    } else {
        // 5..8 bits: the 1024-cell search grid and a single-code table (code -> its fp16 level in the low half)
        if ((st = build_wide_grid(k_bits, t.data(), lut)) != TQ_OK) return st;
        pairs.resize(k);
        for (int i = 0; i < k; ++i) pairs[i] = c16[i];
    }

    tq_codec* c = new tq_codec();
    c->d = d;
    c->bits = k_bits;
    c->seed = seed;
    c->rotation = rotation;
    cudaGetDevice(&c->device);
    auto cleanup = [&](tq_status s) {
        tq_codec_destroy(c);
        return s;
    };
    if (cudaMalloc(&c->pi_op, dd * 2) != cudaSuccess || cudaMalloc(&c->pi_op_t, dd * 2) != cudaSuccess ||
        cudaMalloc(&c->enc_lut, lut.size() * sizeof(uint32_t)) != cudaSuccess ||
        cudaMalloc(&c->pair_lut, pairs.size() * 4) != cudaSuccess)
        return cleanup(fail(TQ_ERR_CUDA, "tq_codec_create: cudaMalloc failed"));
    if (cudaMemcpy(c->pi_op, pi16.data(), dd * 2, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->pi_op_t, pit16.data(), dd * 2, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->enc_lut, lut.data(), lut.size() * sizeof(uint32_t), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->pair_lut, pairs.data(), pairs.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
        return cleanup(fail(TQ_ERR_CUDA, "tq_codec_create: cudaMemcpy failed"));
    if ((st = make_tmap_f16(&c->tmap_pi, c->pi_op, d, d, d, d)) != TQ_OK) return cleanup(st);
    if ((st = make_tmap_f16(&c->tmap_pit, c->pi_op_t, d, d, d, d)) != TQ_OK) return cleanup(st);
    *out = c;
    return TQ_OK;
}

extern "C" tq_status tq_codec_create(int d, int k_bits, uint64_t seed, tq_codec** out) {
    return tq_codec_create_ex(d, k_bits, seed, TQ_ROT_HAAR, out);
}

extern "C" tq_status tq_codec_destroy(tq_codec* c) {
    if (!c) return TQ_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    cudaFree(c->pi_op);
    cudaFree(c->pi_op_t);
    cudaFree(c->enc_lut);
    cudaFree(c->pair_lut);
    cudaFree(c->s_op);
    cudaSetDevice(prev);
    delete c;
    return TQ_OK;
}

extern "C" tq_status tq_codec_create_qjl(int d, int bits, uint64_t seed, int rotation, tq_codec** out) {
    clear_error();
    if (!out) return fail(TQ_ERR_INVALID_ARG, "tq_codec_create_qjl: out is NULL");
    *out = nullptr;
    if (bits < 2 || bits > 5)
        return fail(TQ_ERR_UNSUPPORTED, "tq_codec_create_qjl: bits=%d (supported: 2..5, an MSE stage of bits - 1)", bits);
    tq_codec* c = nullptr;
    tq_status st = tq_codec_create_ex(d, bits - 1, seed, rotation, &c);
    if (st != TQ_OK) return st;
    // S: Gaussian draws i * d + j of the generator seeded with seed + 10000; the tensor cores multiply by fp16(S)
    const size_t dd = static_cast<size_t>(d) * d;
    std::vector<double> sg(dd);
    host_gaussians(seed + kQjlSeedOffset, dd, sg.data());
    std::vector<uint16_t> s16(dd);
    double row_max = 0.0;
    for (int i = 0; i < d; ++i) {
        double ss = 0.0;
        for (int j = 0; j < d; ++j) {
            s16[static_cast<size_t>(i) * d + j] = f64_to_f16(sg[static_cast<size_t>(i) * d + j]);
            const double v = f16_to_f64(s16[static_cast<size_t>(i) * d + j]);
            ss += v * v;
        }
        row_max = std::max(row_max, std::sqrt(ss));
    }
    c->s_row_max = static_cast<float>(row_max * (1.0 + 1e-6));
    if (cudaMalloc(&c->s_op, dd * 2) != cudaSuccess ||
        cudaMemcpy(c->s_op, s16.data(), dd * 2, cudaMemcpyHostToDevice) != cudaSuccess) {
        tq_codec_destroy(c);
        return fail(TQ_ERR_CUDA, "tq_codec_create_qjl: upload of the sketch failed");
    }
    c->qjl_bits = bits;
    *out = c;
    return TQ_OK;
}

extern "C" tq_status tq_codec_qjl_bits(const tq_codec* c, int* bits) {
    clear_error();
    if (!c || !bits) return fail(TQ_ERR_INVALID_ARG, "tq_codec_qjl_bits: codec and bits must be non-NULL");
    *bits = c->qjl_bits;
    return TQ_OK;
}

extern "C" tq_status tq_codec_info(const tq_codec* c, int* d, int* k_bits, uint64_t* seed) {
    clear_error();
    if (!c) return fail(TQ_ERR_INVALID_ARG, "tq_codec_info: codec is NULL");
    if (d) *d = c->d;
    if (k_bits) *k_bits = c->bits;
    if (seed) *seed = c->seed;
    return TQ_OK;
}

extern "C" tq_status tq_codec_rotation(const tq_codec* c, int* rotation) {
    clear_error();
    if (!c || !rotation) return fail(TQ_ERR_INVALID_ARG, "tq_codec_rotation: codec and rotation must be non-NULL");
    *rotation = c->rotation;
    return TQ_OK;
}

// ---------------------------------------------------------------------------------------- key codec

namespace {

template <int D, int BITS>
tq_status launch_encode_k(const tq_codec* c, const void* x, int64_t n, int64_t stride, const int64_t* slots,
                          uint8_t* packed, float* norms, cudaStream_t st, long long wait_limit = kWaitLimitCycles,
                          int withhold_first_tile = 0) {
    // separate instantiations with and without a slot mapping, so the contiguous one carries none of its code
    static std::atomic<uint64_t> mask_rows{0}, mask_slots{0};
    constexpr uint32_t smem = enc_smem_bytes<D, BITS>();
    auto kern = slots ? encode_k_kernel<D, BITS, true> : encode_k_kernel<D, BITS, false>;
    TQ_CUDA(allow_smem(kern, smem, slots ? mask_slots : mask_rows), "tq_encode_k: cudaFuncSetAttribute");
    CUtensorMap tx;
    tq_status s = make_tmap_f16(&tx, x, static_cast<uint64_t>(n), D, static_cast<uint64_t>(stride), 128);
    if (s != TQ_OK) return s;
    const int64_t tiles = (n + 127) / 128;
    const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
    kern<<<grid, EncCfg<D>::kThreads, smem, st>>>(tx, c->tmap_pi, c->enc_lut, n, slots, packed, norms, wait_limit,
                                                  withhold_first_tile);
    TQ_CUDA(cudaGetLastError(), "tq_encode_k: launch");
    return TQ_OK;
}

template <int D, int BITS>
tq_status launch_decode_k(const tq_codec* c, const uint8_t* packed, const float* norms, int64_t n, void* out,
                          int dtype, cudaStream_t st) {
    static std::atomic<uint64_t> mask16{0}, mask32{0};
    constexpr uint32_t smem = dec_smem_bytes<D, BITS>();
    const int64_t tiles = (n + 127) / 128;
    const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
    CUtensorMap tmap_out;
    tq_status s = make_tmap_out(&tmap_out, out, static_cast<uint64_t>(n), D, dtype == TQ_F32);
    if (s != TQ_OK) return s;
    if (dtype == TQ_F32) {
        auto kern = decode_k_kernel<D, BITS, true>;
        TQ_CUDA(allow_smem(kern, smem, mask32), "tq_decode_k: cudaFuncSetAttribute");
        kern<<<grid, DecCfg<D>::kThreads, smem, st>>>(c->tmap_pit, tmap_out, c->pair_lut, packed, norms, n);
    } else {
        auto kern = decode_k_kernel<D, BITS, false>;
        TQ_CUDA(allow_smem(kern, smem, mask16), "tq_decode_k: cudaFuncSetAttribute");
        kern<<<grid, DecCfg<D>::kThreads, smem, st>>>(c->tmap_pit, tmap_out, c->pair_lut, packed, norms, n);
    }
    TQ_CUDA(cudaGetLastError(), "tq_decode_k: launch");
    return TQ_OK;
}

#define TQ_DISPATCH_DB(d, bits, FN, ...)                                                              \
    switch ((d) * 10 + (bits)) {                                                                      \
        case 641: return FN<64, 1>(__VA_ARGS__);                                                      \
        case 642: return FN<64, 2>(__VA_ARGS__);                                                      \
        case 643: return FN<64, 3>(__VA_ARGS__);                                                      \
        case 644: return FN<64, 4>(__VA_ARGS__);                                                      \
        case 1281: return FN<128, 1>(__VA_ARGS__);                                                    \
        case 1282: return FN<128, 2>(__VA_ARGS__);                                                    \
        case 1283: return FN<128, 3>(__VA_ARGS__);                                                    \
        case 1284: return FN<128, 4>(__VA_ARGS__);                                                    \
        case 2561: return FN<256, 1>(__VA_ARGS__);                                                    \
        case 2562: return FN<256, 2>(__VA_ARGS__);                                                    \
        case 2563: return FN<256, 3>(__VA_ARGS__);                                                    \
        case 2564: return FN<256, 4>(__VA_ARGS__);                                                    \
        case 645: return FN<64, 5>(__VA_ARGS__);                                                      \
        case 646: return FN<64, 6>(__VA_ARGS__);                                                      \
        case 647: return FN<64, 7>(__VA_ARGS__);                                                      \
        case 648: return FN<64, 8>(__VA_ARGS__);                                                      \
        case 1285: return FN<128, 5>(__VA_ARGS__);                                                    \
        case 1286: return FN<128, 6>(__VA_ARGS__);                                                    \
        case 1287: return FN<128, 7>(__VA_ARGS__);                                                    \
        case 1288: return FN<128, 8>(__VA_ARGS__);                                                    \
        default: return fail(TQ_ERR_UNSUPPORTED, "unsupported d=%d bits=%d", (d), (bits));            \
    }

}  // namespace

extern "C" tq_status tq_encode_k(const tq_codec* c, const void* x, int64_t n, int64_t x_row_stride,
                                 const int64_t* slot_mapping, uint8_t* packed, float* norms, void* stream) {
    clear_error();
    if (!c) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: codec is NULL");
    if (n < 0) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: n=%lld is negative", static_cast<long long>(n));
    if (n == 0) return TQ_OK;
    if (n > (1ll << 31) - 256) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: n=%lld exceeds 2^31-256 rows", static_cast<long long>(n));
    if (!x || !packed || !norms) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: x, packed and norms must be non-NULL");
    if (!aligned(x, 16)) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: x must be 16-byte aligned");
    if (x_row_stride < c->d || x_row_stride % 8)
        return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: x_row_stride=%lld must be >= d and a multiple of 8",
                    static_cast<long long>(x_row_stride));
    if (!aligned(packed, 16) || !aligned(norms, 4))
        return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: packed must be 16-byte and norms 4-byte aligned");
    if (slot_mapping && !aligned(slot_mapping, 8)) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k: slot_mapping misaligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TQ_DISPATCH_DB(c->d, c->bits, launch_encode_k, c, x, n, x_row_stride, slot_mapping, packed, norms, st);
}

namespace {

template <int D, int KB>
tq_status launch_qjl_residual(const tq_codec* c, const void* x, int64_t n, int64_t stride, const int64_t* slots,
                              const uint8_t* packed, const float* norms, uint8_t* signs, float* rho, cudaStream_t st) {
    if constexpr (KB > 4) {
        return fail(TQ_ERR_UNSUPPORTED, "tq_encode_k_qjl: an MSE stage of %d bits (QJL codecs have 1..4)", KB);
    } else {
    static std::atomic<uint64_t> mask{0};
    constexpr uint32_t smem = qjl_smem_bytes<D, KB>();
    auto kern = qjl_residual_kernel<D, KB>;
    TQ_CUDA(allow_smem(kern, smem, mask), "tq_encode_k_qjl: cudaFuncSetAttribute");
    constexpr int W = qjl_warps<D>();
    const int64_t grid = (n + 16 * W - 1) / (16 * W);
    kern<<<static_cast<unsigned>(grid), 32 * W, smem, st>>>(static_cast<const __half*>(x), n, stride, slots,
                                                                     packed, norms, c->pair_lut, c->pi_op_t, c->s_op,
                                                                     signs, rho);
    TQ_CUDA(cudaGetLastError(), "tq_encode_k_qjl: residual launch");
    return TQ_OK;
    }
}

}  // namespace

extern "C" tq_status tq_encode_k_qjl(const tq_codec* c, const void* x, int64_t n, int64_t x_row_stride,
                                     const int64_t* slot_mapping, uint8_t* packed, float* norms, uint8_t* signs,
                                     float* rho, void* stream) {
    clear_error();
    if (!c) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k_qjl: codec is NULL");
    if (!c->qjl_bits) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k_qjl: the codec was not made by tq_codec_create_qjl");
    if (n == 0) return TQ_OK;
    if (!signs || !rho) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k_qjl: signs and rho must be non-NULL");
    if (!aligned(rho, 4)) return fail(TQ_ERR_INVALID_ARG, "tq_encode_k_qjl: rho must be 4-byte aligned");
    // the MSE stage: the codec's key encoder at bits - 1 (same checks and formats as tq_encode_k)
    tq_status s = tq_encode_k(c, x, n, x_row_stride, slot_mapping, packed, norms, stream);
    if (s != TQ_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TQ_DISPATCH_DB(c->d, c->bits, launch_qjl_residual, c, x, n, x_row_stride, slot_mapping, packed, norms, signs, rho,
                   st);
}

extern "C" tq_status tq_decode_k(const tq_codec* c, const uint8_t* packed, const float* norms, int64_t n, void* out,
                                 int out_dtype, void* stream) {
    clear_error();
    if (!c) return fail(TQ_ERR_INVALID_ARG, "tq_decode_k: codec is NULL");
    if (n < 0) return fail(TQ_ERR_INVALID_ARG, "tq_decode_k: n=%lld is negative", static_cast<long long>(n));
    if (out_dtype != TQ_F16 && out_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "tq_decode_k: out_dtype=%d", out_dtype);
    if (n == 0) return TQ_OK;
    if (!packed || !norms || !out) return fail(TQ_ERR_INVALID_ARG, "tq_decode_k: packed, norms and out must be non-NULL");
    if (!aligned(packed, 16) || !aligned(norms, 16) || !aligned(out, 16))
        return fail(TQ_ERR_INVALID_ARG, "tq_decode_k: packed, norms and out must be 16-byte aligned");
    if (n > INT32_MAX) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_k: n=%lld rows (at most 2^31 - 1 per call)",
                                   static_cast<long long>(n));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TQ_DISPATCH_DB(c->d, c->bits, launch_decode_k, c, packed, norms, n, out, out_dtype, st);
}

// -------------------------------------------------------------------------------------- value codec

namespace {

// Grid of the value kernels (256 threads, grid-stride over 16-element lane chunks): enough CTAs for the work,
// at most one wave of the kernel's resident CTAs (queried once per device), so the grid never ends in a partial
// wave that leaves the SMs nearly idle (a fixed 16 CTAs per SM ran 3.2 waves: value decode 61.4 -> 59.4 us).
template <auto Kernel>
int grid_for(int64_t units) {
    static std::atomic<int> occupancy[64];
    int dev = 0;
    cudaGetDevice(&dev);
    int occ = occupancy[dev & 63].load();
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, Kernel, 256, 0) != cudaSuccess || occ < 1) occ = 1;
        occupancy[dev & 63].store(occ);
    }
    const int64_t blocks = (units + 255) / 256;
    const int64_t cap = static_cast<int64_t>(sm_count()) * occ;
    return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

template <int D, int BITS, int GROUP>
tq_status launch_encode_v(const void* x, int64_t n, int64_t stride, const int64_t* slots, uint8_t* data, void* scales,
                          void* zeros, cudaStream_t st) {
    encode_v_kernel<D, BITS, GROUP><<<grid_for<encode_v_kernel<D, BITS, GROUP>>(n * (D / 16)), 256, 0, st>>>(
        static_cast<const __half*>(x), n, stride, slots, data, static_cast<__half*>(scales), static_cast<__half*>(zeros));
    TQ_CUDA(cudaGetLastError(), "tq_encode_v: launch");
    return TQ_OK;
}

template <int D, int BITS, int GROUP>
tq_status launch_decode_v(const uint8_t* data, const void* scales, const void* zeros, int64_t n, void* out, int dtype,
                          cudaStream_t st) {
    const int grid = (dtype == TQ_F32) ? grid_for<decode_v_kernel<D, BITS, GROUP, true>>(n * (D / 16))
                                       : grid_for<decode_v_kernel<D, BITS, GROUP, false>>(n * (D / 16));
    if (dtype == TQ_F32)
        decode_v_kernel<D, BITS, GROUP, true><<<grid, 256, 0, st>>>(data, static_cast<const __half*>(scales),
                                                                    static_cast<const __half*>(zeros), n, out);
    else
        decode_v_kernel<D, BITS, GROUP, false><<<grid, 256, 0, st>>>(data, static_cast<const __half*>(scales),
                                                                     static_cast<const __half*>(zeros), n, out);
    TQ_CUDA(cudaGetLastError(), "tq_decode_v: launch");
    return TQ_OK;
}

// dispatch over d in {64,128,256}, bits in {2,3,4,8}, group in {32, d}
#define TQ_V_CASE(D_, B_, FN, ...)                                                                    \
    case D_ * 100 + B_ * 10 + 0: return FN<D_, B_, 32>(__VA_ARGS__);                                  \
    case D_ * 100 + B_ * 10 + 1: return FN<D_, B_, D_>(__VA_ARGS__);
#define TQ_V_D(D_, FN, ...)                                                                           \
    TQ_V_CASE(D_, 2, FN, __VA_ARGS__) TQ_V_CASE(D_, 3, FN, __VA_ARGS__) TQ_V_CASE(D_, 4, FN, __VA_ARGS__) \
    TQ_V_CASE(D_, 8, FN, __VA_ARGS__)
#define TQ_DISPATCH_V(d, bits, group, FN, ...)                                                        \
    switch ((d) * 100 + (bits) * 10 + ((group) == (d) ? 1 : 0)) {                                     \
        TQ_V_D(64, FN, __VA_ARGS__)                                                                   \
        TQ_V_D(128, FN, __VA_ARGS__)                                                                  \
        TQ_V_D(256, FN, __VA_ARGS__)                                                                  \
        default: return fail(TQ_ERR_UNSUPPORTED, "unsupported value format d=%d bits=%d group=%d", (d), (bits), (group)); \
    }

tq_status check_v_format(const char* fn, int d, int bits, int group) {
    if (!supported_d(d)) return fail(TQ_ERR_UNSUPPORTED, "%s: d=%d (supported: 64, 128, 256)", fn, d);
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8)
        return fail(TQ_ERR_UNSUPPORTED, "%s: bits=%d (value bits must be one of 2, 3, 4, 8)", fn, bits);
    if (group != 32 && group != d) return fail(TQ_ERR_UNSUPPORTED, "%s: group=%d (32 or d)", fn, group);
    return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_encode_v(int d, int bits, int group, const void* x, int64_t n, int64_t x_row_stride,
                                 const int64_t* slot_mapping, uint8_t* data, void* scales, void* zeros, void* stream) {
    clear_error();
    tq_status s = check_v_format("tq_encode_v", d, bits, group);
    if (s != TQ_OK) return s;
    if (n < 0) return fail(TQ_ERR_INVALID_ARG, "tq_encode_v: n=%lld is negative", static_cast<long long>(n));
    if (n == 0) return TQ_OK;
    if (!x || !data || !scales || !zeros) return fail(TQ_ERR_INVALID_ARG, "tq_encode_v: NULL pointer argument");
    if (!aligned(x, 16) || x_row_stride < d || x_row_stride % 8)
        return fail(TQ_ERR_INVALID_ARG, "tq_encode_v: x must be 16-byte aligned with x_row_stride >= d, a multiple of 8");
    if (!aligned(data, 16) || !aligned(scales, 2) || !aligned(zeros, 2))
        return fail(TQ_ERR_INVALID_ARG, "tq_encode_v: data must be 16-byte aligned");
    if (slot_mapping && !aligned(slot_mapping, 8)) return fail(TQ_ERR_INVALID_ARG, "tq_encode_v: slot_mapping misaligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TQ_DISPATCH_V(d, bits, group, launch_encode_v, x, n, x_row_stride, slot_mapping, data, scales, zeros, st);
}

extern "C" tq_status tq_decode_v(int d, int bits, int group, const uint8_t* data, const void* scales, const void* zeros,
                                 int64_t n, void* out, int out_dtype, void* stream) {
    clear_error();
    tq_status s = check_v_format("tq_decode_v", d, bits, group);
    if (s != TQ_OK) return s;
    if (n < 0) return fail(TQ_ERR_INVALID_ARG, "tq_decode_v: n=%lld is negative", static_cast<long long>(n));
    if (out_dtype != TQ_F16 && out_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "tq_decode_v: out_dtype=%d", out_dtype);
    if (n == 0) return TQ_OK;
    if (!data || !scales || !zeros || !out) return fail(TQ_ERR_INVALID_ARG, "tq_decode_v: NULL pointer argument");
    if (!aligned(data, 16) || !aligned(out, 16) || !aligned(scales, 2) || !aligned(zeros, 2))
        return fail(TQ_ERR_INVALID_ARG, "tq_decode_v: data and out must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TQ_DISPATCH_V(d, bits, group, launch_decode_v, data, scales, zeros, n, out, out_dtype, st);
}

// ---------------------------------------------------------------------------------------- attention

namespace {

constexpr int kAttendCtasPerSm = 4;

struct AttendPlan {
    int num_splits;
    int num_parts;             // num_splits, + 1 with a window
    size_t qfrag_bytes;        // query fragments, one block per (sequence, kv head)
    size_t partial_bytes;      // split-K partials (0 with one split)
    size_t workspace_bytes;    // qfrag_bytes + partial_bytes
};

// ctas_per_sm: attention CTAs resident per SM.  Workspace sizes are planned with the largest (4); a launch
// re-plans with its kernel's measured occupancy, which never needs more splits, so the workspace suffices.
tq_status plan_attend(const tq_attend_args* a, AttendPlan* plan, bool window = false,
                      int ctas_per_sm = kAttendCtasPerSm, bool qjl = false) {
    if (!a) return fail(TQ_ERR_INVALID_ARG, "tq_attend: args is NULL");
    if (a->batch < 1 || a->num_kv_heads < 1 || a->num_q_heads < 1)
        return fail(TQ_ERR_INVALID_ARG, "tq_attend: batch, num_q_heads, num_kv_heads must be >= 1");
    if (a->num_q_heads % a->num_kv_heads)
        return fail(TQ_ERR_INVALID_ARG, "tq_attend: num_q_heads=%d is not a multiple of num_kv_heads=%d", a->num_q_heads,
                    a->num_kv_heads);
    if (a->num_q_heads / a->num_kv_heads > 8)
        return fail(TQ_ERR_UNSUPPORTED, "tq_attend: GQA group %d > 8", a->num_q_heads / a->num_kv_heads);
    if (!supported_d(a->head_dim)) return fail(TQ_ERR_UNSUPPORTED, "tq_attend: head_dim=%d", a->head_dim);
    tq_status s = check_v_format("tq_attend", a->head_dim, a->v_bits, a->v_group);
    if (s != TQ_OK) return s;
    int64_t max_chunks;
    if (a->block_table) {
        if (a->block_size != 16) return fail(TQ_ERR_UNSUPPORTED, "tq_attend: block_size=%d (supported: 16)", a->block_size);
        if (a->max_blocks < 1) return fail(TQ_ERR_INVALID_ARG, "tq_attend: max_blocks=%d", a->max_blocks);
        if (!a->seq_lens) return fail(TQ_ERR_INVALID_ARG, "tq_attend: the paged layout needs seq_lens");
        max_chunks = a->max_blocks;
    } else {
        if (a->max_seq_len < 0 || a->max_seq_len % 16)
            return fail(TQ_ERR_INVALID_ARG, "tq_attend: max_seq_len=%lld must be a non-negative multiple of 16",
                        static_cast<long long>(a->max_seq_len));
        max_chunks = a->max_seq_len / 16;
    }
    const int64_t bh = static_cast<int64_t>(a->batch) * a->num_kv_heads;
    // fill every SM's resident CTAs at most once (a grid one CTA past the resident slots runs a second, mostly
    // empty wave that costs a whole CTA duration); a window's extra CTA per (sequence, kv head) takes one slot
    int64_t splits = (static_cast<int64_t>(sm_count()) * ctas_per_sm - (window ? bh : 0)) / bh;
    const int64_t by_len = (max_chunks + 7) / 8;            // at least ~8 chunks (128 tokens) per split
    if (splits > by_len) splits = by_len;
    if (splits > kMaxSplits) splits = kMaxSplits;
    if (splits < 1) splits = 1;
    plan->num_splits = static_cast<int>(splits);
    plan->num_parts = static_cast<int>(splits) + (window ? 1 : 0);
    plan->partial_bytes =
        (plan->num_parts > 1) ? static_cast<size_t>(bh) * plan->num_parts * (16 + 8 * a->head_dim) * 4 : 0;
    // prepared query fragments per (sequence, kv head): Pi_op q, and with QJL keys also S_op q
    plan->qfrag_bytes = static_cast<size_t>(bh) * ((a->head_dim / 16) * 32 + 2) * 16 * (qjl ? 2 : 1);
    plan->workspace_bytes = plan->qfrag_bytes + plan->partial_bytes;
    return TQ_OK;
}

template <int D, int KB, int VB, int VG, bool QJL = false>
tq_status launch_attend(const tq_codec* c, const tq_attend_args* a, const tq_attend_window* win,
                        const tq_qjl_keys* qjl, const AttendPlan& plan_max, cudaStream_t st) {
    using Cfg = AttCfg<D, KB, VB, VG, QJL>;
    static std::atomic<uint64_t> mask{0};
    static std::atomic<int> occupancy[64];                // resident CTAs per SM, per device (0: not yet queried)
    auto kern = attend_kernel<D, KB, VB, VG, QJL>;
    TQ_CUDA(allow_smem(kern, Cfg::kSmem, mask), "tq_attend_decode: cudaFuncSetAttribute");
    int dev = 0;
    cudaGetDevice(&dev);
    int occ = occupancy[dev & 63].load();
    if (occ == 0) {
        TQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, Cfg::kThreads, Cfg::kSmem),
                "tq_attend_decode: cudaOccupancyMaxActiveBlocksPerMultiprocessor");
        occ = occ < 1 ? 1 : (occ > kAttendCtasPerSm ? kAttendCtasPerSm : occ);
        occupancy[dev & 63].store(occ);
    }
    // split the sequences so that the grid fills the resident CTAs once
    AttendPlan plan = plan_max;
    if (occ < kAttendCtasPerSm) {
        tq_status s = plan_attend(a, &plan, win != nullptr, occ, QJL);
        if (s != TQ_OK) return s;
    }
    AttendParams p;
    p.batch = a->batch;
    p.num_q_heads = a->num_q_heads;
    p.num_kv_heads = a->num_kv_heads;
    p.group = a->num_q_heads / a->num_kv_heads;
    const float scale = (a->scale == 0.f) ? 1.0f / std::sqrt(static_cast<float>(D)) : a->scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.max_seq_len = a->max_seq_len;
    p.block_table = a->block_table;
    p.max_blocks = a->max_blocks;
    p.seq_lens = a->seq_lens;
    p.q = static_cast<const __half*>(a->q);
    p.pi_op = c->pi_op;
    p.pair_lut = c->pair_lut;
    p.k_packed = a->k_packed;
    p.k_norms = a->k_norms;
    p.v_data = a->v_data;
    p.v_scales = static_cast<const __half*>(a->v_scales);
    p.v_zeros = static_cast<const __half*>(a->v_zeros);
    p.out = a->out;
    p.qfrag = static_cast<uint4*>(a->workspace);
    p.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(a->workspace) + plan.qfrag_bytes);
    p.num_splits = plan.num_splits;
    p.num_parts = plan.num_parts;
    p.win_k = nullptr;
    p.win_v = nullptr;
    p.win_lens = nullptr;
    p.win_max = 0;
    p.qfrag_stride = qfrag_slots<D>() * (QJL ? 2 : 1);
    p.k_signs = QJL ? qjl->signs : nullptr;
    p.k_rho = QJL ? qjl->rho : nullptr;
    p.s_op = c->s_op;
    p.s_scale_log2 = p.scale_log2 * static_cast<float>(std::sqrt(std::acos(-1.0) / 2.0) / D);
    p.s_row_bound = c->s_row_max;
    if (win) {
        p.win_k = static_cast<const __half*>(win->k);
        p.win_v = static_cast<const __half*>(win->v);
        p.win_lens = win->lens;
        p.win_max = win->max_len;
    }
    attend_prep_kernel<D><<<dim3((QJL ? 2 : 1) * D / 32, a->num_kv_heads, a->batch), kPrepThreads, 0, st>>>(p);
    TQ_CUDA(cudaGetLastError(), "tq_attend_decode: query preparation launch");
    // the attention grid and the split merge are programmatic dependents of the grid before them: each is
    // scheduled while its predecessor drains and waits for it (griddepcontrol.wait) before reading its output
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.num_parts, a->num_kv_heads, a->batch);   // split CTAs, then the window's
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TQ_CUDA(cudaLaunchKernelEx(&cfg, kern, p), "tq_attend_decode: launch");
    if (plan.num_parts > 1) {
        cfg.gridDim = dim3(p.group * (D / kMergeCols), a->num_kv_heads, a->batch);
        cfg.blockDim = dim3(kMergeThreads);
        cfg.dynamicSmemBytes = 0;
        TQ_CUDA(cudaLaunchKernelEx(&cfg, attend_merge_kernel<D>, p), "tq_attend_decode: merge launch");
    }
    return TQ_OK;
}

template <int D, int KB>
tq_status attend_v(const tq_codec* c, const tq_attend_args* a, const tq_attend_window* win, const tq_qjl_keys* qjl,
                   const AttendPlan& plan, cudaStream_t st) {
    const bool tok = a->v_group == D;
    if constexpr (KB > 4) {
        // keys of 5..8 bits (e.g. protected layers): values of 2, 4 or 8 bits in groups of 32
        if (!qjl && !tok && a->v_bits == 2) return launch_attend<D, KB, 2, 32>(c, a, win, qjl, plan, st);
        if (!qjl && !tok && a->v_bits == 4) return launch_attend<D, KB, 4, 32>(c, a, win, qjl, plan, st);
        if (!qjl && !tok && a->v_bits == 8) return launch_attend<D, KB, 8, 32>(c, a, win, qjl, plan, st);
        return fail(TQ_ERR_UNSUPPORTED,
                    "tq_attend_decode: keys of %d bits take values of 2, 4 or 8 bits in groups of 32 (v_bits=%d "
                    "v_group=%d)", KB, a->v_bits, a->v_group);
    }
    if (qjl) {
        // QJL residual keys: values of 2 or 4 bits in groups of 32
        if (!tok && a->v_bits == 2) return launch_attend<D, KB, 2, 32, true>(c, a, win, qjl, plan, st);
        if (!tok && a->v_bits == 4) return launch_attend<D, KB, 4, 32, true>(c, a, win, qjl, plan, st);
        return fail(TQ_ERR_UNSUPPORTED, "tq_attend_decode_qjl: v_bits=%d v_group=%d (supported: 2 or 4 bits, group 32)",
                    a->v_bits, a->v_group);
    }
    switch (a->v_bits * 2 + (tok ? 1 : 0)) {
        case 4: return launch_attend<D, KB, 2, 32>(c, a, win, qjl, plan, st);
        case 5: return launch_attend<D, KB, 2, D>(c, a, win, qjl, plan, st);
        case 6: return launch_attend<D, KB, 3, 32>(c, a, win, qjl, plan, st);
        case 7: return launch_attend<D, KB, 3, D>(c, a, win, qjl, plan, st);
        case 8: return launch_attend<D, KB, 4, 32>(c, a, win, qjl, plan, st);
        case 9: return launch_attend<D, KB, 4, D>(c, a, win, qjl, plan, st);
        case 16: return launch_attend<D, KB, 8, 32>(c, a, win, qjl, plan, st);
        case 17: return launch_attend<D, KB, 8, D>(c, a, win, qjl, plan, st);
        default: return fail(TQ_ERR_UNSUPPORTED, "tq_attend_decode: v_bits=%d", a->v_bits);
    }
}

}  // namespace

namespace {

tq_status check_window(const char* fn, const tq_attend_window* w) {
    if (!w) return fail(TQ_ERR_INVALID_ARG, "%s: window is NULL", fn);
    if (w->max_len < 1 || w->max_len > TQ_ATTEND_WINDOW_MAX)
        return fail(TQ_ERR_INVALID_ARG, "%s: window max_len=%d outside 1..%d", fn, w->max_len, TQ_ATTEND_WINDOW_MAX);
    return TQ_OK;
}

tq_status attend_decode_impl(const char* fn, const tq_codec* c, const tq_attend_args* a, const tq_attend_window* win,
                             void* stream, const tq_qjl_keys* qjl = nullptr) {
    if (!c) return fail(TQ_ERR_INVALID_ARG, "%s: codec is NULL", fn);
    AttendPlan plan;
    tq_status s = plan_attend(a, &plan, win != nullptr, kAttendCtasPerSm, qjl != nullptr);
    if (s != TQ_OK) return s;
    if (a->head_dim != c->d) return fail(TQ_ERR_INVALID_ARG, "%s: head_dim=%d but the codec has d=%d", fn, a->head_dim, c->d);
    if (!a->q || !a->k_packed || !a->k_norms || !a->v_data || !a->v_scales || !a->v_zeros || !a->out)
        return fail(TQ_ERR_INVALID_ARG, "%s: NULL pointer in args", fn);
    if (!a->workspace || a->workspace_bytes < plan.workspace_bytes)
        return fail(TQ_ERR_INVALID_ARG, "%s: workspace of %zu bytes required (got %zu)", fn, plan.workspace_bytes,
                    a->workspace ? a->workspace_bytes : static_cast<size_t>(0));
    if (!aligned(a->q, 16) || !aligned(a->k_packed, 16) || !aligned(a->k_norms, 16) || !aligned(a->v_data, 16) ||
        !aligned(a->v_scales, 16) || !aligned(a->v_zeros, 16) || !aligned(a->out, 16) || !aligned(a->workspace, 16))
        return fail(TQ_ERR_INVALID_ARG, "%s: every pointer must be 16-byte aligned", fn);
    if (win) {
        if ((s = check_window(fn, win)) != TQ_OK) return s;
        if (!win->k || !win->v) return fail(TQ_ERR_INVALID_ARG, "%s: window k and v must be non-NULL", fn);
        if (!aligned(win->k, 16) || !aligned(win->v, 16) || (win->lens && !aligned(win->lens, 4)))
            return fail(TQ_ERR_INVALID_ARG, "%s: window k and v must be 16-byte aligned", fn);
    }
    if (qjl) {
        if (!c->qjl_bits) return fail(TQ_ERR_INVALID_ARG, "%s: the codec was not made by tq_codec_create_qjl", fn);
        if (!qjl->signs || !qjl->rho) return fail(TQ_ERR_INVALID_ARG, "%s: signs and rho must be non-NULL", fn);
        if (!aligned(qjl->signs, 16) || !aligned(qjl->rho, 16))
            return fail(TQ_ERR_INVALID_ARG, "%s: signs and rho must be 16-byte aligned", fn);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (c->d * 10 + c->bits) {
        case 641: return attend_v<64, 1>(c, a, win, qjl, plan, st);
        case 642: return attend_v<64, 2>(c, a, win, qjl, plan, st);
        case 643: return attend_v<64, 3>(c, a, win, qjl, plan, st);
        case 644: return attend_v<64, 4>(c, a, win, qjl, plan, st);
        case 1281: return attend_v<128, 1>(c, a, win, qjl, plan, st);
        case 1282: return attend_v<128, 2>(c, a, win, qjl, plan, st);
        case 1283: return attend_v<128, 3>(c, a, win, qjl, plan, st);
        case 1284: return attend_v<128, 4>(c, a, win, qjl, plan, st);
        case 2561: return attend_v<256, 1>(c, a, win, qjl, plan, st);
        case 2562: return attend_v<256, 2>(c, a, win, qjl, plan, st);
        case 2563: return attend_v<256, 3>(c, a, win, qjl, plan, st);
        case 2564: return attend_v<256, 4>(c, a, win, qjl, plan, st);
        case 645: return attend_v<64, 5>(c, a, win, qjl, plan, st);
        case 646: return attend_v<64, 6>(c, a, win, qjl, plan, st);
        case 647: return attend_v<64, 7>(c, a, win, qjl, plan, st);
        case 648: return attend_v<64, 8>(c, a, win, qjl, plan, st);
        case 1285: return attend_v<128, 5>(c, a, win, qjl, plan, st);
        case 1286: return attend_v<128, 6>(c, a, win, qjl, plan, st);
        case 1287: return attend_v<128, 7>(c, a, win, qjl, plan, st);
        case 1288: return attend_v<128, 8>(c, a, win, qjl, plan, st);
        default: return fail(TQ_ERR_UNSUPPORTED, "%s: d=%d bits=%d", fn, c->d, c->bits);
    }
}

}  // namespace

namespace {

template <int D, int KB>
tq_status launch_scores(const tq_codec* c, const tq_attend_args* a, const AttendPlan& plan, float* scores,
                        int64_t score_len, cudaStream_t st) {
    static std::atomic<uint64_t> mask{0};
    auto kern = attend_scores_kernel<D, KB>;
    const uint32_t smem = 2u * static_cast<uint32_t>(key_table_entries<KB>()) * 128u;
    TQ_CUDA(allow_smem(kern, smem, mask), "tq_attend_scores: cudaFuncSetAttribute");
    AttendParams p = {};
    p.batch = a->batch;
    p.num_q_heads = a->num_q_heads;
    p.num_kv_heads = a->num_kv_heads;
    p.group = a->num_q_heads / a->num_kv_heads;
    const float scale = (a->scale == 0.f) ? 1.0f / std::sqrt(static_cast<float>(D)) : a->scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.max_seq_len = a->max_seq_len;
    p.block_table = a->block_table;
    p.max_blocks = a->max_blocks;
    p.seq_lens = a->seq_lens;
    p.q = static_cast<const __half*>(a->q);
    p.pi_op = c->pi_op;
    p.pair_lut = c->pair_lut;
    p.k_packed = a->k_packed;
    p.k_norms = a->k_norms;
    p.qfrag = static_cast<uint4*>(a->workspace);
    p.num_splits = p.num_parts = 1;
    p.qfrag_stride = qfrag_slots<D>();
    p.k_signs = nullptr;
    p.k_rho = nullptr;
    p.s_op = nullptr;
    p.s_scale_log2 = 0.f;
    p.s_row_bound = 0.f;
    attend_prep_kernel<D><<<dim3(D / 32, a->num_kv_heads, a->batch), kPrepThreads, 0, st>>>(p);
    TQ_CUDA(cudaGetLastError(), "tq_attend_scores: query preparation launch");
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((score_len + 63) / 64), a->num_kv_heads, a->batch);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TQ_CUDA(cudaLaunchKernelEx(&cfg, kern, p, scores, score_len), "tq_attend_scores: launch");
    return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_attend_scores(const tq_codec* c, const tq_attend_args* a, float* scores, void* stream) {
    clear_error();
    if (!c) return fail(TQ_ERR_INVALID_ARG, "tq_attend_scores: codec is NULL");
    AttendPlan plan;
    tq_status s = plan_attend(a, &plan);
    if (s != TQ_OK) return s;
    if (a->head_dim != c->d) return fail(TQ_ERR_INVALID_ARG, "tq_attend_scores: head_dim=%d but the codec has d=%d", a->head_dim, c->d);
    if (!a->q || !a->k_packed || !a->k_norms || !scores)
        return fail(TQ_ERR_INVALID_ARG, "tq_attend_scores: q, k_packed, k_norms and scores must be non-NULL");
    if (!a->workspace || a->workspace_bytes < plan.qfrag_bytes)
        return fail(TQ_ERR_INVALID_ARG, "tq_attend_scores: workspace of %zu bytes required (got %zu)", plan.qfrag_bytes,
                    a->workspace ? a->workspace_bytes : static_cast<size_t>(0));
    if (!aligned(a->q, 16) || !aligned(a->k_norms, 4) || !aligned(a->workspace, 16) || !aligned(scores, 4))
        return fail(TQ_ERR_INVALID_ARG, "tq_attend_scores: q and workspace must be 16-byte aligned");
    const int64_t score_len = a->block_table ? static_cast<int64_t>(a->max_blocks) * 16 : a->max_seq_len;
    if (score_len == 0) return TQ_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TQ_DISPATCH_DB(c->d, c->bits, launch_scores, c, a, plan, scores, score_len, st);
}

extern "C" tq_status tq_attend_workspace_bytes(const tq_attend_args* a, size_t* bytes) {
    clear_error();
    if (!bytes) return fail(TQ_ERR_INVALID_ARG, "tq_attend_workspace_bytes: bytes is NULL");
    *bytes = 0;
    AttendPlan plan;
    tq_status s = plan_attend(a, &plan);
    if (s != TQ_OK) return s;
    *bytes = plan.workspace_bytes;
    return TQ_OK;
}

extern "C" tq_status tq_attend_qjl_workspace_bytes(const tq_attend_args* a, size_t* bytes) {
    clear_error();
    if (!bytes) return fail(TQ_ERR_INVALID_ARG, "tq_attend_qjl_workspace_bytes: bytes is NULL");
    *bytes = 0;
    AttendPlan plan;
    tq_status s = plan_attend(a, &plan, false, kAttendCtasPerSm, true);
    if (s != TQ_OK) return s;
    *bytes = plan.workspace_bytes;
    return TQ_OK;
}

extern "C" tq_status tq_attend_decode_qjl(const tq_codec* c, const tq_attend_args* a, const tq_qjl_keys* keys,
                                          void* stream) {
    clear_error();
    if (!keys) return fail(TQ_ERR_INVALID_ARG, "tq_attend_decode_qjl: keys is NULL");
    return attend_decode_impl("tq_attend_decode_qjl", c, a, nullptr, stream, keys);
}

extern "C" tq_status tq_attend_window_workspace_bytes(const tq_attend_args* a, const tq_attend_window* w, size_t* bytes) {
    clear_error();
    if (!bytes) return fail(TQ_ERR_INVALID_ARG, "tq_attend_window_workspace_bytes: bytes is NULL");
    *bytes = 0;
    tq_status s = check_window("tq_attend_window_workspace_bytes", w);
    if (s != TQ_OK) return s;
    AttendPlan plan;
    if ((s = plan_attend(a, &plan, true)) != TQ_OK) return s;
    *bytes = plan.workspace_bytes;
    return TQ_OK;
}

extern "C" tq_status tq_attend_decode(const tq_codec* c, const tq_attend_args* a, void* stream) {
    clear_error();
    return attend_decode_impl("tq_attend_decode", c, a, nullptr, stream);
}

extern "C" tq_status tq_attend_decode_window(const tq_codec* c, const tq_attend_args* a, const tq_attend_window* w,
                                             void* stream) {
    clear_error();
    if (!w) return fail(TQ_ERR_INVALID_ARG, "tq_attend_decode_window: window is NULL");
    return attend_decode_impl("tq_attend_decode_window", c, a, w, stream);
}

// ---------------------------------------------------------------------- attention without allocation

// Scratch for tq_attend_decode_noalloc: part of this library's device image, so it exists on every device
// that loads the library, without any allocation call by the entry point.
static __device__ __align__(256) unsigned char g_attend_scratch[TQ_ATTEND_SCRATCH_BYTES];

namespace {

// Device address of g_attend_scratch on the current device, looked up once per device.  In host code the
// array's name is only a stand-in, never a device address, so kernels must receive this pointer.
tq_status attend_scratch(void** out) {
    static std::mutex mu;
    static std::vector<void*> addr;
    int dev = 0;
    TQ_CUDA(cudaGetDevice(&dev), "tq_attend_decode_noalloc: cudaGetDevice");
    std::lock_guard<std::mutex> lk(mu);
    if (static_cast<int>(addr.size()) <= dev) addr.resize(dev + 1, nullptr);
    if (!addr[dev]) {
        void* p = nullptr;
        TQ_CUDA(cudaGetSymbolAddress(&p, g_attend_scratch), "tq_attend_decode_noalloc: cudaGetSymbolAddress");
        addr[dev] = p;
    }
    *out = addr[dev];
    return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_attend_decode_noalloc(const tq_codec* c, const tq_attend_args* a, void* stream) {
    clear_error();
    if (!c) return fail(TQ_ERR_INVALID_ARG, "tq_attend_decode_noalloc: codec is NULL");
    AttendPlan plan;
    tq_status s = plan_attend(a, &plan);
    if (s != TQ_OK) return s;
    if (plan.workspace_bytes > TQ_ATTEND_SCRATCH_BYTES)
        return fail(TQ_ERR_INVALID_ARG,
                    "tq_attend_decode_noalloc: this launch needs %zu bytes of scratch but the static scratch "
                    "holds %u; use tq_attend_decode with a workspace",
                    plan.workspace_bytes, TQ_ATTEND_SCRATCH_BYTES);
    void* scratch = nullptr;
    if ((s = attend_scratch(&scratch)) != TQ_OK) return s;
    tq_attend_args with_scratch = *a;
    with_scratch.workspace = scratch;
    with_scratch.workspace_bytes = TQ_ATTEND_SCRATCH_BYTES;
    return tq_attend_decode(c, &with_scratch, stream);
}

// --------------------------------------------------------------------------------------- diagnostics

extern "C" tq_status tq_stream_status(void* stream, int clear) {
    clear_error();
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned v = 0;
    TQ_CUDA(cudaMemcpyFromSymbolAsync(&v, g_error_flag, sizeof(v), 0, cudaMemcpyDeviceToHost, st),
            "tq_stream_status: read");
    TQ_CUDA(cudaStreamSynchronize(st), "tq_stream_status: cudaStreamSynchronize");
    if (v && clear) {
        const unsigned z = 0;
        TQ_CUDA(cudaMemcpyToSymbolAsync(g_error_flag, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st),
                "tq_stream_status: clear");
        TQ_CUDA(cudaStreamSynchronize(st), "tq_stream_status: cudaStreamSynchronize");
    }
    if (v) return fail(TQ_ERR_DEVICE_FLAG, "a kernel's bounded wait expired (device flag 0x%x)", v);
    return TQ_OK;
}

extern "C" tq_status tq_debug_encode_k_stalled(const tq_codec* c, const void* x, int64_t n, uint8_t* packed,
                                               float* norms, long long wait_limit_cycles, void* stream) {
    clear_error();
    if (!c) return fail(TQ_ERR_INVALID_ARG, "tq_debug_encode_k_stalled: codec is NULL");
    if (n < 1 || n > (1ll << 31) - 256) return fail(TQ_ERR_INVALID_ARG, "tq_debug_encode_k_stalled: n=%lld", (long long)n);
    if (wait_limit_cycles < 1000 || wait_limit_cycles > kWaitLimitCycles)
        return fail(TQ_ERR_INVALID_ARG, "tq_debug_encode_k_stalled: wait_limit_cycles=%lld outside [1000, %lld]",
                    wait_limit_cycles, static_cast<long long>(kWaitLimitCycles));
    if (!x || !packed || !norms || !aligned(x, 16) || !aligned(packed, 16) || !aligned(norms, 4))
        return fail(TQ_ERR_INVALID_ARG, "tq_debug_encode_k_stalled: x, packed and norms must be non-NULL and aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TQ_DISPATCH_DB(c->d, c->bits, launch_encode_k, c, x, n, c->d, nullptr, packed, norms, st, wait_limit_cycles, 1);
}

extern "C" tq_status tq_read_device_flag(int* flag_out, int clear) {
    clear_error();
    if (!flag_out) return fail(TQ_ERR_INVALID_ARG, "tq_read_device_flag: flag_out is NULL");
    TQ_CUDA(cudaDeviceSynchronize(), "tq_read_device_flag: cudaDeviceSynchronize");
    unsigned v = 0;
    TQ_CUDA(cudaMemcpyFromSymbol(&v, g_error_flag, sizeof(v)), "tq_read_device_flag: read");
    *flag_out = static_cast<int>(v);
    if (clear) {
        unsigned z = 0;
        TQ_CUDA(cudaMemcpyToSymbol(g_error_flag, &z, sizeof(z)), "tq_read_device_flag: clear");
    }
    return TQ_OK;
}
