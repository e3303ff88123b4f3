// Encode / decode kernels for keys (rotated Lloyd-Max, tcgen05) and values (grouped affine).
#pragma once

#include "tq_device.cuh"

namespace tq {
namespace dev {

// --------------------------------------------------------------------------------- bit-field helpers

// OR value v (< 2^BITS) into the little-endian bitstream `w` at field j (compile-time after unrolling).
template <int BITS, int NW>
__device__ __forceinline__ void put_field(uint32_t (&w)[NW], int j, uint32_t v) {
    const int bit = j * BITS, wi = bit >> 5, sh = bit & 31;
    w[wi] |= v << sh;
    if (sh + BITS > 32) w[wi + 1] |= v >> (32 - sh);
}

// Field of width W starting at bit `bit` of the little-endian bitstream `w`.
template <int W, int NW>
__device__ __forceinline__ uint32_t get_bits(const uint32_t (&w)[NW], int bit) {
    const int wi = bit >> 5, sh = bit & 31;
    uint32_t v = w[wi] >> sh;
    if (sh + W > 32) v |= w[wi + 1] << (32 - sh);
    return (W == 32) ? v : (v & ((1u << W) - 1u));
}

// Store NW words (4-byte aligned destination; wider vectors where NW allows and `dst` is aligned to them).
template <int NW>
__device__ __forceinline__ void store_words(uint8_t* dst, const uint32_t (&w)[NW]) {
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 4)
            *reinterpret_cast<uint4*>(dst + 4 * i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
    } else if constexpr (NW == 2) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) reinterpret_cast<uint32_t*>(dst)[i] = w[i];
    }
}

template <int NW>
__device__ __forceinline__ void load_words(const uint8_t* src, uint32_t (&w)[NW]) {
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 4) {
            uint4 v = *reinterpret_cast<const uint4*>(src + 4 * i);
            w[i] = v.x; w[i + 1] = v.y; w[i + 2] = v.z; w[i + 3] = v.w;
        }
    } else if constexpr (NW == 2) {
        uint2 v = *reinterpret_cast<const uint2*>(src);
        w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = reinterpret_cast<const uint32_t*>(src)[i];
    }
}

// ------------------------------------------------------------------------------------ value codec
// "KV Cache API", values.py quantize_values / dequantize_values.  One thread owns one 32-element unit of
// a row (a whole group when GROUP == 32); with GROUP == D the D/32 units of a row sit in consecutive
// lanes and reduce min/max with shuffles.  Every step is the page's fp32 operation, rounded once.

template <int D, int BITS, int GROUP>
__global__ void __launch_bounds__(256) encode_v_kernel(const __half* __restrict__ x, int64_t n, int64_t stride,
                                                       const int64_t* __restrict__ slots, uint8_t* __restrict__ data,
                                                       __half* __restrict__ scales, __half* __restrict__ zeros) {
    constexpr int kUnits = D / 32;
    constexpr int kRowBytes = D * BITS / 8;
    constexpr int kGroups = D / GROUP;
    constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
    const int64_t total = n * kUnits;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    // warp-uniform trip count so every lane takes part in the shuffles
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31); base < total; base += step) {
        const int64_t u = base + (threadIdx.x & 31);
        const bool valid = u < total;
        const int64_t row = valid ? u / kUnits : 0;
        const int part = static_cast<int>(u % kUnits);
        float v[32];
        if (valid) {
            const uint4* p = reinterpret_cast<const uint4*>(x + row * stride + part * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 w = __ldg(p + i);
                const __half2* h = reinterpret_cast<const __half2*>(&w);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float2 f = __half22float2(h[k]);
                    v[8 * i + 2 * k] = f.x;
                    v[8 * i + 2 * k + 1] = f.y;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        float vmin = v[0], vmax = v[0];
#pragma unroll
        for (int i = 1; i < 32; ++i) {
            vmin = fminf(vmin, v[i]);
            vmax = fmaxf(vmax, v[i]);
        }
        if constexpr (GROUP == D) {
#pragma unroll
            for (int off = 1; off < kUnits; off <<= 1) {
                vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, off));
                vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
            }
        }
        float scale = __fdiv_rn(__fsub_rn(vmax, vmin), kLevels);
        scale = fmaxf(scale, 1e-12f);
        const float zero = vmin;
        uint32_t w[BITS];
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            float q = rintf(__fdiv_rn(__fsub_rn(v[i], zero), scale));
            q = fminf(fmaxf(q, 0.f), kLevels);
            put_field<BITS>(w, i, static_cast<uint32_t>(q));
        }
        if (valid) {
            const int64_t orow = slots ? slots[row] : row;
            if (orow >= 0) {
                store_words<BITS>(data + orow * kRowBytes + part * 4 * BITS, w);
                if (GROUP == 32 || part == 0) {
                    const int gi = (GROUP == 32) ? part : 0;
                    scales[orow * kGroups + gi] = __float2half_rn(scale);
                    zeros[orow * kGroups + gi] = __float2half_rn(zero);
                }
            }
        }
    }
}

template <int D, int BITS, int GROUP, bool OUT_F32>
__global__ void __launch_bounds__(256) decode_v_kernel(const uint8_t* __restrict__ data, const __half* __restrict__ scales,
                                                       const __half* __restrict__ zeros, int64_t n, void* __restrict__ out) {
    constexpr int kUnits = D / 32;
    constexpr int kRowBytes = D * BITS / 8;
    constexpr int kGroups = D / GROUP;
    const int64_t total = n * kUnits;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < total; u += step) {
        const int64_t row = u / kUnits;
        const int part = static_cast<int>(u % kUnits);
        uint32_t w[BITS];
        load_words<BITS>(data + row * kRowBytes + part * 4 * BITS, w);
        const int gi = (GROUP == 32) ? part : 0;
        const float s = __half2float(scales[row * kGroups + gi]);
        const float z = __half2float(zeros[row * kGroups + gi]);
        float y[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t q = get_bits<BITS>(w, i * BITS);
            y[i] = __fadd_rn(__fmul_rn(static_cast<float>(q), s), z);
        }
        if constexpr (OUT_F32) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + row * D + part * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
        } else {
            uint4* o = reinterpret_cast<uint4*>(static_cast<__half*>(out) + row * D + part * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 pk;
                __half2 h0 = __floats2half2_rn(y[8 * i], y[8 * i + 1]);
                __half2 h1 = __floats2half2_rn(y[8 * i + 2], y[8 * i + 3]);
                __half2 h2 = __floats2half2_rn(y[8 * i + 4], y[8 * i + 5]);
                __half2 h3 = __floats2half2_rn(y[8 * i + 6], y[8 * i + 7]);
                pk.x = *reinterpret_cast<uint32_t*>(&h0);
                pk.y = *reinterpret_cast<uint32_t*>(&h1);
                pk.z = *reinterpret_cast<uint32_t*>(&h2);
                pk.w = *reinterpret_cast<uint32_t*>(&h3);
                o[i] = pk;
            }
        }
    }
}

// -------------------------------------------------------------------------------------- key codec
// Tiles of 128 vectors.  The d x d rotation is one UMMA chain per tile: D[128 x d] (TMEM, fp32) =
// X[128 x d] (smem, fp16, 128B-swizzled K-major) * B^T with B = Pi_op for encode and Pi_op^T for decode.
// Roles per CTA: warp 0 = TMA producer, warp 1 = TMEM allocator + single-thread MMA issuer,
// warps 2..9 = epilogue (warp w reads TMEM lanes 32*(w%4).. and handles one half of the columns).

template <int D>
struct KeyCfg {
    static constexpr int kRows = 128;
    static constexpr int kKB = D / 64;                       // 128-byte column blocks per row
    static constexpr int kTileBytes = kRows * D * 2;         // one fp16 tile
    static constexpr int kTileBlockBytes = kRows * 128;      // one 64-column block of a tile
    static constexpr int kPiBytes = D * D * 2;
    static constexpr int kPiBlockBytes = D * 128;            // one 64-column block of the d x d matrix
    static constexpr int kEncStages = (D == 256) ? 1 : (D == 128 ? 4 : 6);
    static constexpr int kDecBufs = (D == 256) ? 1 : 2;
    static constexpr int kEpiWarps = 8;
    static constexpr int kThreads = 32 * (2 + kEpiWarps);
    static constexpr int kTmemCols = 2 * D;                  // two accumulator buffers
    static constexpr int kHalfCols = D / 2;
    static constexpr int kChunks = kHalfCols / 32;           // 32-column TMEM loads per thread per tile
    static constexpr int kLutEntries = 2048;                 // encode grid table
    static constexpr uint32_t kIdesc = idesc_f16_f32(128, D);
};

// Encode-side search: y maps to grid cell rint(512 y + 640) (an exact FMA into the 1.5*2^23 magic
// range); the cell's entry holds the count L of boundaries below the cell and the one boundary B that
// may fall inside it (+inf if none): index = L + (y > B).
constexpr float kGridScale = 512.0f;
constexpr float kGridMagic = 12583552.0f;   // 1.5 * 2^23 + 640

struct EncSmem {
    uint32_t pi, x, lut, norm, bar;
};

template <int D>
__host__ __device__ constexpr uint32_t enc_smem_bytes() {
    using C = KeyCfg<D>;
    return C::kPiBytes + C::kEncStages * C::kTileBytes + C::kLutEntries * 8 + 2 * 2 * 128 * 4 +
           8 * (2 * C::kEncStages + 8) + 16 + 1024;
}

template <int D, int BITS>
__global__ void __launch_bounds__(KeyCfg<D>::kThreads, 1)
    encode_k_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_pi,
                    const uint2* __restrict__ lut_g, int64_t n, const int64_t* __restrict__ slots,
                    uint8_t* __restrict__ packed, float* __restrict__ norms) {
    using C = KeyCfg<D>;
    constexpr int S = C::kEncStages;
    constexpr int kRowBytes = D * BITS / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* s_pi = smem;
    uint8_t* s_x = s_pi + C::kPiBytes;
    uint2* s_lut = reinterpret_cast<uint2*>(s_x + S * C::kTileBytes);
    float* s_norm = reinterpret_cast<float*>(s_lut + C::kLutEntries);          // [2 bufs][2 halves][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_norm + 2 * 2 * 128);
    // barrier slots
    const uint32_t b_xfull = smem_u32(bars), b_xempty = b_xfull + 8 * S, b_accfull = b_xempty + 8 * S,
                   b_accempty = b_accfull + 16, b_pifull = b_accempty + 16, b_normrdy = b_pifull + 8,
                   b_final = b_normrdy + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t num_tiles = (n + 127) / 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(b_xfull + 8 * s, 1);
            mbar_init(b_xempty + 8 * s, 1 + C::kEpiWarps);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(b_accfull + 8 * a, 1);
            mbar_init(b_accempty + 8 * a, C::kEpiWarps);
            mbar_init(b_normrdy + 8 * a, C::kEpiWarps);
        }
        mbar_init(b_pifull, 1);
        mbar_init(b_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i < C::kLutEntries; i += blockDim.x) s_lut[i] = lut_g[i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- TMA producer
            mbar_arrive_expect_tx(b_pifull, C::kPiBytes);
            for (int kb = 0; kb < C::kKB; ++kb)
                tma_load_2d(smem_u32(s_pi + kb * C::kPiBlockBytes), &tmap_pi, b_pifull, kb * 64, 0);
            int li = 0;
            for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++li) {
                const int s = li % S;
                const uint32_t ph = (li / S) & 1;
                if (!mbar_wait(b_xempty + 8 * s, ph ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(b_xfull + 8 * s, C::kTileBytes);
                for (int kb = 0; kb < C::kKB; ++kb)
                    tma_load_2d(smem_u32(s_x + s * C::kTileBytes + kb * C::kTileBlockBytes), &tmap_x, b_xfull + 8 * s,
                                kb * 64, static_cast<int>(tile * 128));
            }
            // drain: every issued load has landed before the CTA may exit
            for (int k = (li > S ? li - S : 0); k < li; ++k) mbar_wait_drain(b_xfull + 8 * (k % S), (k / S) & 1);
            mbar_wait_drain(b_pifull, 0);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            bool ok = mbar_wait(b_pifull, 0, abort_flag);
            int li = 0;
            for (int64_t tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++li) {
                const int s = li % S, a = li & 1;
                if (!mbar_wait(b_xfull + 8 * s, (li / S) & 1, abort_flag)) break;
                if (!mbar_wait(b_accempty + 8 * a, ((li >> 1) & 1) ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + a * D;
                const uint32_t xa = smem_u32(s_x + s * C::kTileBytes), pa = smem_u32(s_pi);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k & 3) * 32;
                    const uint64_t ad = desc_kmajor_sw128(xa + (k >> 2) * C::kTileBlockBytes + off);
                    const uint64_t bd = desc_kmajor_sw128(pa + (k >> 2) * C::kPiBlockBytes + off);
                    umma_f16_ss(d_tmem, ad, bd, C::kIdesc, k > 0 ? 1u : 0u);
                }
                umma_commit(b_accfull + 8 * a);
                umma_commit(b_xempty + 8 * s);
            }
            // every MMA has completed before TMEM is released
            umma_commit(b_final);
            mbar_wait_drain(b_final, 0);
        }
    } else {
        // -------------------------------------------------------------------- epilogue
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        const int r = quarter * 32 + lane;
        int li = 0;
        for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++li) {
            const int s = li % S, a = li & 1, nb = li & 1;
            if (!mbar_wait(b_xfull + 8 * s, (li / S) & 1, abort_flag)) break;
            // sum of squares of this half of row r (squares of fp16 values are exact in fp32)
            const uint8_t* xs = s_x + s * C::kTileBytes;
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
            for (int c = 0; c < C::kHalfCols / 8; ++c) {
                const int col = half * C::kHalfCols + c * 8;
                const uint4 v = *reinterpret_cast<const uint4*>(xs + (col >> 6) * C::kTileBlockBytes +
                                                                sw128_offset(r, (col & 63) >> 3));
                const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f = __half22float2(h[k]);
                    acc[2 * k] = fmaf(f.x, f.x, acc[2 * k]);
                    acc[2 * k + 1] = fmaf(f.y, f.y, acc[2 * k + 1]);
                }
            }
            const float part = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
            __syncwarp();
            if (lane == 0) mbar_arrive(b_xempty + 8 * s);
            s_norm[nb * 256 + half * 128 + r] = part;
            __syncwarp();
            if (lane == 0) mbar_arrive(b_normrdy + 8 * nb);
            if (!mbar_wait(b_normrdy + 8 * nb, (li >> 1) & 1, abort_flag)) break;
            const float nrm = sqrtf(s_norm[nb * 256 + r] + s_norm[nb * 256 + 128 + r]);
            const float inv = 1.0f / (nrm + 1e-8f);
            const int64_t row = tile * 128 + r;
            int64_t orow = -1;
            if (row < n) orow = slots ? slots[row] : row;
            if (half == 0 && orow >= 0) norms[orow] = nrm;

            if (!mbar_wait(b_accfull + 8 * a, (li >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * D + half * C::kHalfCols;
#pragma unroll
            for (int ch = 0; ch < C::kChunks; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + ch * 32, v);
                tmem_ld_wait();
                uint32_t w[BITS];
#pragma unroll
                for (int i = 0; i < BITS; ++i) w[i] = 0u;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float y = __uint_as_float(v[j]) * inv;
                    const float g = fmaf(y, kGridScale, kGridMagic);
                    const uint2 e = s_lut[__float_as_uint(g) & (C::kLutEntries - 1)];
                    const uint32_t idx = e.y + (y > __uint_as_float(e.x) ? 1u : 0u);
                    put_field<BITS>(w, j, idx);
                }
                if (orow >= 0)
                    store_words<BITS>(packed + orow * kRowBytes + (half * C::kHalfCols + ch * 32) * BITS / 8, w);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_accempty + 8 * a);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

template <int D>
__host__ __device__ constexpr uint32_t dec_smem_bytes() {
    using C = KeyCfg<D>;
    return C::kPiBytes + C::kDecBufs * C::kTileBytes + 256 * 4 + 8 * (2 * C::kDecBufs + 8) + 16 + 1024;
}

template <int D, int BITS, bool OUT_F32>
__global__ void __launch_bounds__(KeyCfg<D>::kThreads, 1)
    decode_k_kernel(const __grid_constant__ CUtensorMap tmap_pit, const uint32_t* __restrict__ pair_lut_g,
                    const uint8_t* __restrict__ packed, const float* __restrict__ norms, int64_t n,
                    void* __restrict__ out) {
    using C = KeyCfg<D>;
    constexpr int NB = C::kDecBufs;
    constexpr int kRowBytes = D * BITS / 8;
    constexpr int kHalfWords = kRowBytes / 8;      // 32-bit words in half a packed row
    constexpr int kPairs = 1 << (2 * BITS);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* s_pit = smem;
    uint8_t* s_a = s_pit + C::kPiBytes;
    uint32_t* s_pair = reinterpret_cast<uint32_t*>(s_a + NB * C::kTileBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_pair + 256);
    const uint32_t b_afull = smem_u32(bars), b_aempty = b_afull + 8 * NB, b_accfull = b_aempty + 8 * NB,
                   b_accempty = b_accfull + 16, b_pifull = b_accempty + 16, b_final = b_pifull + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NB + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t num_tiles = (n + 127) / 128;

    if (threadIdx.x == 0) {
        for (int b = 0; b < NB; ++b) {
            mbar_init(b_afull + 8 * b, C::kEpiWarps);
            mbar_init(b_aempty + 8 * b, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(b_accfull + 8 * a, 1);
            mbar_init(b_accempty + 8 * a, C::kEpiWarps);
        }
        mbar_init(b_pifull, 1);
        mbar_init(b_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i < kPairs; i += blockDim.x) s_pair[i] = pair_lut_g[i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(b_pifull, C::kPiBytes);
            for (int kb = 0; kb < C::kKB; ++kb)
                tma_load_2d(smem_u32(s_pit + kb * C::kPiBlockBytes), &tmap_pit, b_pifull, kb * 64, 0);
            mbar_wait_drain(b_pifull, 0);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            bool ok = mbar_wait(b_pifull, 0, abort_flag);
            int li = 0;
            for (int64_t tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++li) {
                const int b = li % NB, a = li & 1;
                if (!mbar_wait(b_afull + 8 * b, (li / NB) & 1, abort_flag)) break;
                if (!mbar_wait(b_accempty + 8 * a, ((li >> 1) & 1) ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + a * D;
                const uint32_t aa = smem_u32(s_a + b * C::kTileBytes), pa = smem_u32(s_pit);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k & 3) * 32;
                    const uint64_t ad = desc_kmajor_sw128(aa + (k >> 2) * C::kTileBlockBytes + off);
                    const uint64_t bd = desc_kmajor_sw128(pa + (k >> 2) * C::kPiBlockBytes + off);
                    umma_f16_ss(d_tmem, ad, bd, C::kIdesc, k > 0 ? 1u : 0u);
                }
                umma_commit(b_accfull + 8 * a);
                umma_commit(b_aempty + 8 * b);
            }
            umma_commit(b_final);
            mbar_wait_drain(b_final, 0);
        }
    } else {
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        const int r = quarter * 32 + lane;

        // build the A tile (c_op[idx] as fp16, 128B-swizzled K-major) for local tile index lt
        auto build = [&](int lt, int64_t tile) -> bool {
            const int b = lt % NB;
            if (!mbar_wait(b_aempty + 8 * b, ((lt / NB) & 1) ^ 1, abort_flag)) return false;
            const int64_t row = tile * 128 + r;
            uint32_t w[kHalfWords];
            if (row < n) {
                load_words<kHalfWords>(packed + row * kRowBytes + half * (kRowBytes / 2), w);
            } else {
#pragma unroll
                for (int i = 0; i < kHalfWords; ++i) w[i] = 0u;
            }
            uint8_t* as = s_a + b * C::kTileBytes;
#pragma unroll
            for (int c = 0; c < C::kHalfCols / 8; ++c) {
                uint32_t h[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) h[p] = s_pair[get_bits<2 * BITS>(w, (c * 8 + 2 * p) * BITS)];
                const int col = half * C::kHalfCols + c * 8;
                *reinterpret_cast<uint4*>(as + (col >> 6) * C::kTileBlockBytes + sw128_offset(r, (col & 63) >> 3)) =
                    make_uint4(h[0], h[1], h[2], h[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_afull + 8 * b);
            return true;
        };

        bool ok = true;
        int64_t tile = blockIdx.x;
        if (tile < num_tiles) ok = build(0, tile);
        int li = 0;
        for (; ok && tile < num_tiles; tile += gridDim.x, ++li) {
            const int64_t next = tile + gridDim.x;
            if (next < num_tiles && !build(li + 1, next)) break;
            const int a = li & 1;
            const int64_t row = tile * 128 + r;
            const float nrm = (row < n) ? norms[row] : 0.f;
            if (!mbar_wait(b_accfull + 8 * a, (li >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * D + half * C::kHalfCols;
#pragma unroll
            for (int ch = 0; ch < C::kChunks; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + ch * 32, v);
                tmem_ld_wait();
                if (row < n) {
                    const int col = half * C::kHalfCols + ch * 32;
                    if constexpr (OUT_F32) {
                        float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + row * D + col);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            o[i] = make_float4(__uint_as_float(v[4 * i]) * nrm, __uint_as_float(v[4 * i + 1]) * nrm,
                                               __uint_as_float(v[4 * i + 2]) * nrm, __uint_as_float(v[4 * i + 3]) * nrm);
                    } else {
                        uint4* o = reinterpret_cast<uint4*>(static_cast<__half*>(out) + row * D + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint32_t pk[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                __half2 h2 = __floats2half2_rn(__uint_as_float(v[8 * i + 2 * k]) * nrm,
                                                               __uint_as_float(v[8 * i + 2 * k + 1]) * nrm);
                                pk[k] = *reinterpret_cast<uint32_t*>(&h2);
                            }
                            o[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_accempty + 8 * a);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace dev
}  // namespace tq
