// Encode / decode kernels for keys (rotated Lloyd-Max, tcgen05) and values (grouped affine).
#pragma once

#include "tq_device.cuh"

namespace tq {
namespace dev {

// Grid of the key encoder's nearest-level search (built on the host, see tq_lib.cu build_grid_lut):
// kGridCells cells of width 1 / kGridRes; u = kGridRes * y + kGridOffset is rounded to a multiple of 2^-7 and
// the cell is its integer part.
constexpr int kGridRes = 64;
constexpr int kGridOffset = 128;
constexpr int kGridCells = 256;
// Keys of 5..8 bits: a 1024-cell grid of 8-byte entries (boundary, count below), built by tq_lib.cu
// build_wide_grid; cell = bits 5..14 of fma(sat(fma(y, s, 0.5)), 1023.75, 1.5 * 2^18).  Each entry is stored
// kWideCopies times side by side and lane l reads copy l % kWideCopies, which spreads a warp's lookups of nearby
// cells over more banks.
constexpr int kWideCells = 1024;
constexpr int kWideCopies = 4;
constexpr int kWideWords = 2 * kWideCells * kWideCopies + 4;   // the entries, then s (padded to 16 bytes)

// ------------------------------------------------------------------------------------ value codec
// "KV Cache API", values.py quantize_values / dequantize_values.  The lanes of one scale group reduce
// min/max with shuffles.  Every arithmetic step is the page's fp32 operation with one rounding.

// Codes of a group: round_half_even(a / s) with the page's IEEE fp32 division, 0 <= a <= (2^b - 1) s.
// With r an approximate reciprocal of s (relative error <= 2^-21; the hardware's is about 2^-23), the
// products a RN(r (1 -+ 2^-20)) bracket both a / s and RN(a / s): each end lies at least 2^-21 (a/s) away
// from a / s on its side, beyond the half ulp (<= 2^-24 (a/s)) that separates a / s from RN(a / s).  An FMA
// adding 1.5 * 2^23 rounds each end to the nearest integer (ties to even) in its low mantissa bits.  Rounding
// is monotonic, so when both ends give the same integer, RN(a / s) rounds to it as well; otherwise the caller
// recomputes with the exact quotient.
constexpr float kCodeMagic = 12582912.0f;                   // 1.5 * 2^23
constexpr uint32_t kCodeMagicBits = 0x4B400000u;

// RN(x / L) for x >= 0 and L in {3, 7, 15, 255}: q = RN(x RN(1/L)), then one correction step with the exact
// residual x - q L computed by an FMA -- the quotient correction of Markstein's method (P. Markstein, "IA-64
// and Elementary Functions", 2000; the residual of a product is exact under an FMA), applied once to a constant
// divisor.  Checked exhaustively against IEEE division for every non-negative finite fp32 x and each of the
// four L (all 2^31 - 2^23 values, on the host with hardware FMA).
template <int L>
__device__ __forceinline__ float div_by_levels(float x) {
    constexpr float y = 1.0f / static_cast<float>(L);
    const float q = __fmul_rn(x, y);
    return __fmaf_rn(__fmaf_rn(-q, static_cast<float>(L), x), y, q);
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// One lane owns 16 consecutive elements of a row (32 bytes of fp16), so a group of 32 spans 2 lanes (or d/16
// lanes in the per-token layout), the per-group division and reciprocal of the encoder are shared by 16
// elements, and every warp-wide load and store covers whole rows.
template <int D, int GROUP>
struct VLanes {
    static constexpr int kRowLanes = D / 16;
    static constexpr int kRowsPerWarp = 32 / kRowLanes;           // 2, 4 or 8
    static constexpr int kGroupLanes = GROUP / 16;                // 2 or d/16
};

// f32(h) - c with one rounding (h exact in f32, so this is the page's fp32 subtraction of the fp16 input)
__device__ __forceinline__ float sub_f16_f32(__half h, float c) {
    float d;
    asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(__half_as_ushort(h)), "f"(c));
    return d;
}

// sum_k kMagicBits * 2^(BITS k) over the codes packed into one 32-bit word (mod 2^32): packing the raw bits
// of the rounded values (kCodeMagicBits + code) with multiply-adds leaves exactly this constant on top
template <int BITS>
__host__ __device__ constexpr uint32_t magic_pack_offset() {
    uint32_t c = 0u;
    for (int k = 0; k < 32 / BITS; ++k) c += kCodeMagicBits << (BITS * k);
    return c;
}

template <int D, int BITS, int GROUP>
__global__ void __launch_bounds__(256) encode_v_kernel(const __half* __restrict__ x, int64_t n, int64_t stride,
                                                       const int64_t* __restrict__ slots, uint8_t* __restrict__ data,
                                                       __half* __restrict__ scales, __half* __restrict__ zeros) {
    using L = VLanes<D, GROUP>;
    constexpr int kRowBytes = D * BITS / 8;
    constexpr int kGroups = D / GROUP;
    constexpr uint32_t kLevels = (1u << BITS) - 1u;
    constexpr int kW = (16 * BITS + 31) / 32;                     // words holding this lane's 16 codes
    constexpr bool kWordAligned = (32 % BITS == 0);               // codes never straddle a word (2, 4, 8 bits)
    const int lane = threadIdx.x & 31;
    const int j = lane % L::kRowLanes;                            // 16-element chunk index within the row
    const int gl = j % L::kGroupLanes;                            // lane index within the scale group
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    const int64_t step = warps_total * L::kRowsPerWarp;
    // this lane's 16 inputs of row r (zeros past n); the next row's are loaded before the current one is encoded
    auto load = [&](int64_t r, uint4& w0, uint4& w1) {
        if (r < n) {
            const uint4* src = reinterpret_cast<const uint4*>(x + r * stride) + 2 * j;
            w0 = __ldg(src);
            w1 = __ldg(src + 1);
        } else {
            w0 = w1 = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    int64_t wrow = (static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5)) * L::kRowsPerWarp;
    uint4 c0, c1;
    load(wrow + lane / L::kRowLanes, c0, c1);
    for (; wrow < n; wrow += step) {
        const int64_t row = wrow + lane / L::kRowLanes;
        const bool valid = row < n;
        uint4 n0, n1;
        load(row + step, n0, n1);
        __half2 hv[8];
        {
            const uint32_t u[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) hv[k] = *reinterpret_cast<const __half2*>(&u[k]);
        }
        c0 = n0;
        c1 = n1;
        // min / max on packed halves (exact; fp16 -> fp32 is exact afterwards)
        __half2 mn2 = __hmin2(hv[0], hv[1]), mx2 = __hmax2(hv[0], hv[1]);
#pragma unroll
        for (int k = 2; k < 8; ++k) {
            mn2 = __hmin2(mn2, hv[k]);
            mx2 = __hmax2(mx2, hv[k]);
        }
        float vmin = fminf(__low2float(mn2), __high2float(mn2));
        float vmax = fmaxf(__low2float(mx2), __high2float(mx2));
#pragma unroll
        for (int off = 1; off < L::kGroupLanes; off <<= 1) {
            vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, off));
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
        }
        float scale = div_by_levels<static_cast<int>(kLevels)>(__fsub_rn(vmax, vmin));   // = IEEE (max - min) / L
        scale = fmaxf(scale, 1e-12f);                                 // a normal number from here on
        const float zero = vmin;
        const float rcp = rcp_approx(scale);
        const float r_lo = __fmul_rn(rcp, 0.99999904632568359375f);   // 1 - 2^-20
        const float r_hi = __fmul_rn(rcp, 1.00000095367431640625f);   // 1 + 2^-20
        uint32_t chunk[kW];
#pragma unroll
        for (int k = 0; k < kW; ++k) chunk[k] = 0u;
        uint32_t differ = 0u;
        const float2 rlo2 = make_float2(r_lo, r_lo), rhi2 = make_float2(r_hi, r_hi);
        const float2 mag2 = make_float2(kCodeMagic, kCodeMagic);
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) {
            // two elements per packed f32x2 FMA (each lane of the pair is the scalar IEEE operation)
            const float2 a = make_float2(sub_f16_f32(__low2half(hv[k2]), zero), sub_f16_f32(__high2half(hv[k2]), zero));
            const float2 lo2 = __ffma2_rn(a, rlo2, mag2), hi2 = __ffma2_rn(a, rhi2, mag2);
            const uint32_t tlo[2] = {__float_as_uint(lo2.x), __float_as_uint(lo2.y)};
            differ |= (tlo[0] ^ __float_as_uint(hi2.x)) | (tlo[1] ^ __float_as_uint(hi2.y));
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int k = 2 * k2 + e;
                // the code never exceeds 2^b - 1 (a <= max - min), so the low bits of tlo are the code and the
                // bits above are the constant kCodeMagicBits
                if constexpr (kWordAligned) {
                    constexpr int kPer = 32 / BITS;
                    chunk[k / kPer] += tlo[e] << (BITS * (k % kPer));   // shift-add; the magic is removed below
                } else {
                    put_field<BITS>(chunk, k, tlo[e] & kLevels);
                }
            }
        }
        if constexpr (kWordAligned) {
#pragma unroll
            for (int k = 0; k < kW; ++k) chunk[k] -= magic_pack_offset<BITS>();
        }
        if (differ != 0u) {
#pragma unroll
            for (int k = 0; k < kW; ++k) chunk[k] = 0u;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const __half hk = (k & 1) ? __high2half(hv[k >> 1]) : __low2half(hv[k >> 1]);
                const float q = rintf(__fdiv_rn(sub_f16_f32(hk, zero), scale));
                put_field<BITS>(chunk, k, static_cast<uint32_t>(fminf(fmaxf(q, 0.f), static_cast<float>(kLevels))));
            }
        }
        const int64_t orow = valid ? (slots ? slots[row] : row) : -1;
        uint8_t* dst = data + orow * kRowBytes;
        if constexpr (BITS == 2) {
            if (orow >= 0) reinterpret_cast<uint32_t*>(dst)[j] = chunk[0];
        } else if constexpr (BITS == 4) {
            if (orow >= 0) reinterpret_cast<uint2*>(dst)[j] = make_uint2(chunk[0], chunk[1]);
        } else if constexpr (BITS == 8) {
            if (orow >= 0) reinterpret_cast<uint4*>(dst)[j] = make_uint4(chunk[0], chunk[1], chunk[2], chunk[3]);
        } else {
            // 3 bits: 16 codes = 48 bits = 3 half-words at byte 6j (2-byte aligned)
            if (orow >= 0) {
                uint16_t* h = reinterpret_cast<uint16_t*>(dst + 6 * j);
                h[0] = static_cast<uint16_t>(chunk[0]);
                h[1] = static_cast<uint16_t>(chunk[0] >> 16);
                h[2] = static_cast<uint16_t>(chunk[1]);
            }
        }
        if (orow >= 0 && gl == 0) {
            const int gi = j / L::kGroupLanes;
            scales[orow * kGroups + gi] = __float2half_rn(scale);
            zeros[orow * kGroups + gi] = __float2half_rn(zero);
        }
    }
}

// The 16 codes (16 BITS bits) of 16-element chunk j of a value row.
template <int D, int BITS>
__device__ __forceinline__ void load_vchunk16(const uint8_t* src, int j, uint32_t (&c)[4]) {
    if constexpr (BITS == 2) {
        c[0] = __ldg(reinterpret_cast<const uint32_t*>(src) + j);
    } else if constexpr (BITS == 4) {
        const uint2 t = __ldg(reinterpret_cast<const uint2*>(src) + j);
        c[0] = t.x; c[1] = t.y;
    } else if constexpr (BITS == 8) {
        const uint4 t = __ldg(reinterpret_cast<const uint4*>(src) + j);
        c[0] = t.x; c[1] = t.y; c[2] = t.z; c[3] = t.w;
    } else {
        // 48 bits at byte 6j (2-byte aligned)
        const uint16_t* h = reinterpret_cast<const uint16_t*>(src) + 3 * j;
        c[0] = static_cast<uint32_t>(__ldg(h)) | (static_cast<uint32_t>(__ldg(h + 1)) << 16);
        c[1] = __ldg(h + 2);
    }
}

// Decode: one lane owns 16 consecutive elements of a row, so a warp's rows are one contiguous block of 512
// output elements.  The lane writes its 16 results to the warp's shared-memory buffer and one lane sends the
// block to global memory with a bulk copy (double-buffered), so the output bypasses the load/store queue; the
// next rows' codes, scale and zero are loaded before the current rows are converted.
template <int D, int BITS, int GROUP, bool OUT_F32>
__global__ void __launch_bounds__(256) decode_v_kernel(const uint8_t* __restrict__ data, const __half* __restrict__ scales,
                                                       const __half* __restrict__ zeros, int64_t n, void* __restrict__ out) {
    using L = VLanes<D, GROUP>;
    constexpr int kRowBytes = D * BITS / 8;
    constexpr int kGroups = D / GROUP;
    constexpr int kElt = OUT_F32 ? 4 : 2;
    constexpr int kBlockBytes = 32 * 16 * kElt;                    // one warp iteration of output
    __shared__ __align__(128) uint8_t s_out[8][2][kBlockBytes];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = lane % L::kRowLanes;
    const int gi = j / L::kGroupLanes;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    const int64_t step = warps_total * L::kRowsPerWarp;
    int64_t wrow = (static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + warp) * L::kRowsPerWarp;
    const int rl = lane / L::kRowLanes;
    // codes, scale and zero of the rows kPf iterations ahead are in flight while the current rows convert
    // (one iteration: two measured slower with the permute path, the extra registers cost occupancy)
    constexpr int kPf = 1;
    uint32_t c[kPf + 1][4];
    __half s16[kPf + 1], z16[kPf + 1];
#pragma unroll
    for (int f = 0; f <= kPf; ++f) {
        const int64_t frow = wrow + f * step + rl;
        c[f][0] = c[f][1] = c[f][2] = c[f][3] = 0u;
        s16[f] = z16[f] = __float2half_rn(0.f);
        if (f < kPf && frow < n) {
            load_vchunk16<D, BITS>(data + frow * kRowBytes, j, c[f]);
            s16[f] = __ldg(scales + frow * kGroups + gi);
            z16[f] = __ldg(zeros + frow * kGroups + gi);
        }
    }
    for (int it = 0; wrow < n; wrow += step, ++it) {
        const int64_t nrow = wrow + kPf * step + rl;
        if (nrow < n) {
            load_vchunk16<D, BITS>(data + nrow * kRowBytes, j, c[kPf]);
            s16[kPf] = __ldg(scales + nrow * kGroups + gi);
            z16[kPf] = __ldg(zeros + nrow * kGroups + gi);
        }
        const float s = __half2float(s16[0]), z = __half2float(z16[0]);
        const int buf = it & 1;
        if (it >= 2) {
            if (lane == 0) bulk_wait_read<1>();                      // the copy that last read this buffer is done
            __syncwarp();
        }
        uint8_t* sb = &s_out[warp][buf][0];
        // q * s is exact in fp32 (q < 2^8, s an fp16), so (2^23 + q) s - 2^23 s in one FMA is exactly q s and the
        // page's two roundings reduce to the one of the final addition: y = RN(RN(q s) + z) = RN(q s + z)
        const float2 s2 = make_float2(s, s), z2 = make_float2(z, z);
        const float2 off2 = make_float2(-8388608.0f * s, -8388608.0f * s);
        if constexpr (BITS == 2 && !OUT_F32) {
            // the four possible outputs of the lane's group, fp16(RN(q s + z)) for q = 0..3, by the same
            // operations, as two half2 registers; each output pair is one byte permute of them, its selector
            // (2 qa, 2 qa + 1, 2 qb, 2 qb + 1) one multiply-add of the codes spread to bytes 0 and 1
            const float2 y01 = __fadd2_rn(__ffma2_rn(make_float2(__uint_as_float(0x4B000000u), __uint_as_float(0x4B000001u)),
                                                     s2, off2), z2);
            const float2 y23 = __fadd2_rn(__ffma2_rn(make_float2(__uint_as_float(0x4B000002u), __uint_as_float(0x4B000003u)),
                                                     s2, off2), z2);
            __half2 h01 = __floats2half2_rn(y01.x, y01.y), h23 = __floats2half2_rn(y23.x, y23.y);
            const uint32_t t0 = *reinterpret_cast<uint32_t*>(&h01), t1 = *reinterpret_cast<uint32_t*>(&h23);
            const uint32_t ev = c[0][0] & 0x33333333u, od = (c[0][0] >> 2) & 0x33333333u;  // codes 2k, 2k + 1 in nibble k
            uint32_t pk[8];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t wm = __byte_perm(ev, od, 0x40u + m + (m << 4));   // byte 0: ev.m, byte 1: od.m
                const uint32_t lo = wm & 0x0303u, hi = (wm >> 4) & 0x0303u;
                pk[2 * m] = __byte_perm(t0, t1, lo * 0x22u + 0x1010u);
                pk[2 * m + 1] = __byte_perm(t0, t1, hi * 0x22u + 0x1010u);
            }
            uint4* o = reinterpret_cast<uint4*>(sb) + 2 * lane;
            o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
            float y[16];
#pragma unroll
            for (int k2 = 0; k2 < 8; ++k2) {
                const float2 qm = make_float2(__uint_as_float(0x4B000000u | get_bits<BITS>(c[0], 2 * k2 * BITS)),
                                              __uint_as_float(0x4B000000u | get_bits<BITS>(c[0], (2 * k2 + 1) * BITS)));
                const float2 yy = __fadd2_rn(__ffma2_rn(qm, s2, off2), z2);
                y[2 * k2] = yy.x;
                y[2 * k2 + 1] = yy.y;
            }
            if constexpr (OUT_F32) {
                float4* o = reinterpret_cast<float4*>(sb) + 4 * lane;
#pragma unroll
                for (int k = 0; k < 4; ++k) o[k] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
            } else {
                uint32_t pk[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    __half2 hh = __floats2half2_rn(y[2 * k], y[2 * k + 1]);
                    pk[k] = *reinterpret_cast<uint32_t*>(&hh);
                }
                uint4* o = reinterpret_cast<uint4*>(sb) + 2 * lane;
                o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            const int64_t rows = (n - wrow < L::kRowsPerWarp) ? n - wrow : L::kRowsPerWarp;
            bulk_store(static_cast<uint8_t*>(out) + wrow * D * kElt, smem_u32(sb), static_cast<uint32_t>(rows * D * kElt));
            bulk_commit();
        }
#pragma unroll
        for (int f = 0; f < kPf; ++f) {
#pragma unroll
            for (int k = 0; k < 4; ++k) c[f][k] = c[f + 1][k];
            s16[f] = s16[f + 1];
            z16[f] = z16[f + 1];
        }
    }
    if (lane == 0) bulk_wait_all();
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
    static constexpr int kLutEntries = kGridCells;           // encode grid table, replicated once per bank
    static constexpr bool kEncStaged = (D <= 128);           // packed output staged for a bulk store
    static constexpr uint32_t kIdesc = idesc_f16_f32(128, D);
};

// Encode-side search: one FMA g = 64 y + (1.5 * 2^16 + 128) rounds u = 64 y + 128 to a multiple of 2^-7 (the
// float's ulp in [2^16, 2^17)), so bits 7..14 of g hold the cell (the integer part of the rounded u) already
// shifted into place for a table entry of 128 bytes; the cell's entry holds the count L of boundaries below the
// cell and the one boundary B that may fall inside it (+inf if none): index = L + (y > B).
constexpr float kGridScale = static_cast<float>(kGridRes);
constexpr float kGridMagic = 98304.0f + kGridOffset;   // 1.5 * 2^16 + 128



// Encode CTA: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-5 compute the row norms of
// each X stage ahead of the epilogue (one row per thread), warps 6.. are the epilogue (kEpiWarps: warp w
// reads TMEM lanes 32*(w%4).. and owns kCols columns of them).
template <int D>
struct EncCfg {
    static constexpr int kNormWarps = 4;                     // one row per norm thread: the norms keep ahead
    static constexpr int kNormRows = 128 / (32 * kNormWarps);   // rows per norm thread per tile
    static constexpr int kEpiWarps = (D == 64) ? 8 : 16;
    static constexpr int kFirstEpi = 2 + kNormWarps;
    static constexpr int kThreads = 32 * (kFirstEpi + kEpiWarps);
    static constexpr int kCols = D * 4 / kEpiWarps;          // columns per epilogue warp: 32, 32, 64
    static constexpr int kChunks = kCols / 32;
};

template <int D, int BITS>
struct EncLayout {
    using C = KeyCfg<D>;
    static constexpr int kRowBytes = D * BITS / 8;
    static constexpr int kPkBytes = C::kEncStaged ? 128 * kRowBytes : 0;   // one staged packed tile
    // input stages: three at d = 128 (room for the aligned grid table, or for the wider tables of 5..8 bits)
    static constexpr int kStages = (D == 128) ? 3 : C::kEncStages;
    // search table: the 256-cell grid up to 4 bits, replicated once per bank; from 5 bits the 1024-cell grid of
    // 8-byte entries (one copy, 8 KB)
    static constexpr int kLutEntries = C::kLutEntries;
    static constexpr uint32_t kPi = 0;
    static constexpr uint32_t kX = kPi + C::kPiBytes;
    static constexpr uint32_t kLut = kX + kStages * C::kTileBytes;
    // entry e of lane l at 128 e + 4 l; up to d = 128 the 32 KB grid table starts on a multiple of its size
    // (slack reserved), so an entry's address is (the cell bits of g, already at bits 7..14) | lane bits: one LOP3
    static constexpr bool kAlignLut = (BITS <= 4 && D <= 128);
    static constexpr uint32_t kLutBytes = (BITS > 4) ? kWideWords * 4 : kLutEntries * 128 * (kAlignLut ? 2 : 1);
    static constexpr uint32_t kPk = kLut + kLutBytes;
    static constexpr uint32_t kNorm = kPk + 2 * kPkBytes;                   // [stage][128] {norm, 1/(norm+1e-8)}
    static constexpr uint32_t kBar = kNorm + kStages * 128 * 8;
    static constexpr int kBars = 4 * kStages + 10;
    static constexpr uint32_t kMisc = kBar + 8 * kBars;
    static constexpr uint32_t kBytes = kMisc + 16 + 1024;                  // + alignment slack
    static_assert(kBytes <= 227 * 1024, "encode layout exceeds the shared memory of one CTA");
};

template <int D, int BITS>
__host__ __device__ constexpr uint32_t enc_smem_bytes() {
    return EncLayout<D, BITS>::kBytes;
}

template <int D, int BITS, bool SLOTS>
__global__ void __launch_bounds__(EncCfg<D>::kThreads, 1)
    encode_k_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_pi,
                    const uint32_t* __restrict__ lut_g, int64_t n, const int64_t* __restrict__ slots,
                    uint8_t* __restrict__ packed, float* __restrict__ norms, long long wait_limit = kWaitLimitCycles,
                    int withhold_first_tile = 0) {
    using C = KeyCfg<D>;
    using E = EncCfg<D>;
    using Lo = EncLayout<D, BITS>;
    constexpr int S = Lo::kStages;
    constexpr int kRowBytes = Lo::kRowBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);   // stays a shared-space pointer
    uint8_t* s_pi = smem + Lo::kPi;
    uint8_t* s_x = smem + Lo::kX;
    uint8_t* s_pk = smem + Lo::kPk;
    float2* s_norm = reinterpret_cast<float2*>(smem + Lo::kNorm);
    const uint32_t bar0 = smem_u32(smem + Lo::kBar);
    const uint32_t b_xfull = bar0, b_xempty = b_xfull + 8 * S, b_nrdy = b_xempty + 8 * S, b_nfree = b_nrdy + 8 * S,
                   b_accfull = b_nfree + 8 * S, b_accempty = b_accfull + 16, b_pifull = b_accempty + 16,
                   b_final = b_pifull + 8, b_pkfull = b_final + 8, b_pkempty = b_pkfull + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lo::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t num_tiles = (n + 127) / 128;
    // SLOTS: this instantiation writes rows through the slot mapping (the host passes slots != nullptr)
    constexpr bool staged = C::kEncStaged && !SLOTS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(b_xfull + 8 * s, 1);
            mbar_init(b_xempty + 8 * s, 1 + E::kNormWarps);
            mbar_init(b_nrdy + 8 * s, E::kNormWarps);
            mbar_init(b_nfree + 8 * s, E::kEpiWarps);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(b_accfull + 8 * a, 1);
            mbar_init(b_accempty + 8 * a, E::kEpiWarps);
            mbar_init(b_pkfull + 8 * a, E::kEpiWarps);
            mbar_init(b_pkempty + 8 * a, 1);
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
    const uint32_t lut_base = Lo::kAlignLut ? (smem_u32(smem + Lo::kLut) + 32767u) & ~32767u : smem_u32(smem + Lo::kLut);
    if constexpr (BITS > 4) {
        uint32_t* tab = reinterpret_cast<uint32_t*>(smem + Lo::kLut);
        for (int i = threadIdx.x; i < kWideWords; i += blockDim.x) tab[i] = __ldg(lut_g + i);
    } else {
        fill_replicated(reinterpret_cast<uint32_t*>(smem + (lut_base - smem_u32(smem))), lut_g, Lo::kLutEntries);
    }
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
                if (!mbar_wait(b_xempty + 8 * s, ((li / S) & 1) ^ 1, abort_flag, wait_limit)) break;
                // test hook: the first tile's copy is never issued (nor its bytes expected), so every wait on it
                // runs out after wait_limit cycles with nothing in flight; the normal launch passes 0
                if (withhold_first_tile && li == 0) continue;
                mbar_arrive_expect_tx(b_xfull + 8 * s, C::kTileBytes);
                for (int kb = 0; kb < C::kKB; ++kb)
                    tma_load_2d(smem_u32(s_x + s * C::kTileBytes + kb * C::kTileBlockBytes), &tmap_x, b_xfull + 8 * s,
                                kb * 64, static_cast<int>(tile * 128));
            }
            for (int k = (li > S ? li - S : 0); k < li; ++k) mbar_wait_drain(b_xfull + 8 * (k % S), (k / S) & 1, wait_limit);
            mbar_wait_drain(b_pifull, 0, wait_limit);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            bool ok = mbar_wait(b_pifull, 0, abort_flag, wait_limit);
            int li = 0;
            for (int64_t tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++li) {
                const int s = li % S, a = li & 1;
                if (!mbar_wait(b_xfull + 8 * s, (li / S) & 1, abort_flag, wait_limit)) break;
                if (!mbar_wait(b_accempty + 8 * a, ((li >> 1) & 1) ^ 1, abort_flag, wait_limit)) break;
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
            umma_commit(b_final);
            mbar_wait_drain(b_final, 0, wait_limit);
        }
    } else if (warp < E::kFirstEpi) {
        // -------------------------------------------------------------------- row norms, ahead of the epilogue
        const int t = (warp - 2) * 32 + lane;                 // rows t, t + 32 kNormWarps, ... of each tile
        int li = 0;
        for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++li) {
            const int s = li % S;
            if (!mbar_wait(b_xfull + 8 * s, (li / S) & 1, abort_flag, wait_limit)) break;
            if (!mbar_wait(b_nfree + 8 * s, ((li / S) & 1) ^ 1, abort_flag, wait_limit)) break;
            const uint8_t* xs = s_x + s * C::kTileBytes;
#pragma unroll
            for (int hrow = 0; hrow < E::kNormRows; ++hrow) {
                const int r = t + 32 * E::kNormWarps * hrow;
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 8
                for (int c = 0; c < D / 8; ++c) {
                    // squares of fp16 values are exact in fp32; eight partial sums keep the rounding small
                    const uint4 v = *reinterpret_cast<const uint4*>(xs + (c >> 3) * C::kTileBlockBytes + sw128_offset(r, c & 7));
                    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        acc[2 * k] = fma_f16_f32(static_cast<uint16_t>(u[k]), acc[2 * k]);
                        acc[2 * k + 1] = fma_f16_f32(static_cast<uint16_t>(u[k] >> 16), acc[2 * k + 1]);
                    }
                }
                const float nrm = sqrtf(((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
                s_norm[s * 128 + r] = make_float2(nrm, 1.0f / (nrm + 1e-8f));
                // with a slot mapping the epilogue stores the norm (it loads the row's slot anyway, a tile ahead of
                // its use); a load of the slot here would stall the norm warps on a global round trip every tile
                const int64_t row = tile * 128 + r;
                if (!SLOTS && row < n) norms[row] = nrm;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(b_xempty + 8 * s);
                mbar_arrive(b_nrdy + 8 * s);
            }
        }
    } else {
        // -------------------------------------------------------------------- epilogue
        const int ew = warp - E::kFirstEpi;
        const int quarter = warp & 3;
        const int c0 = (ew >> 2) * E::kCols;                  // first column of this warp
        const int r = quarter * 32 + lane;
        const bool issuer = (ew == 0 && lane == 0);           // issues the bulk stores of staged tiles
        const uint32_t lut_lane = lut_base + 4u * lane;        // this lane's copy of the search table (its own bank)
        // 5..8 bits: the wide grid's scale s (after the table's entries) and this lane's copy of the entries
        const float wide_s = (BITS > 4) ? __uint_as_float(lds_u32(lut_base + 8u * kWideCells * kWideCopies)) : 0.f;
        const uint32_t wide_lane = lut_base + 8u * static_cast<uint32_t>(lane % kWideCopies);
        int li = 0;
        for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++li) {
            const int s = li % S, a = li & 1, pb = li & 1;
            if (!mbar_wait(b_nrdy + 8 * s, (li / S) & 1, abort_flag, wait_limit)) break;
            const float inv = s_norm[s * 128 + r].y;
            __syncwarp();
            // with a slot mapping the norm entry is read again (and stored) at the end of the tile, so the stage's
            // norms are released there
            if (!SLOTS && lane == 0) mbar_arrive(b_nfree + 8 * s);
            const int64_t row = tile * 128 + r;
            int64_t orow = -1;
            if (!staged && row < n) orow = SLOTS ? slots[row] : row;

            if (!mbar_wait(b_accfull + 8 * a, (li >> 1) & 1, abort_flag, wait_limit)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * D + c0;
            uint8_t* pk = s_pk + pb * Lo::kPkBytes + r * kRowBytes;
            if (staged && !mbar_wait(b_pkempty + 8 * pb, ((li >> 1) & 1) ^ 1, abort_flag, wait_limit)) break;
#pragma unroll
            for (int k = 0; k < E::kChunks; ++k) {
                uint32_t w[BITS];
#pragma unroll
                for (int i = 0; i < BITS; ++i) w[i] = 0u;
                const float2 inv2 = make_float2(inv, inv);
                const float2 gs2 = make_float2(kGridScale, kGridScale), gm2 = make_float2(kGridMagic, kGridMagic);
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + k * 32, v);
                tmem_ld_wait();
                if (k == E::kChunks - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_accempty + 8 * a);   // TMEM buffer a is free for tile li + 2
                }
#pragma unroll
                for (int j2 = 0; j2 < 16; ++j2) {
                    // two coordinates per packed f32x2 multiply and FMA
                    const float2 y2 = __fmul2_rn(make_float2(__uint_as_float(v[2 * j2]), __uint_as_float(v[2 * j2 + 1])), inv2);
                    const float2 g2 = __ffma2_rn(y2, gs2, gm2);
                    const float yv[2] = {y2.x, y2.y};
                    const uint32_t cell[2] = {__float_as_uint(g2.x), __float_as_uint(g2.y)};
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        if constexpr (BITS > 4) {
                            // 5..8 bits: the 1024-cell grid (cell = bits 5..14 of the second FMA, so the offset of
                            // its group of kWideCopies 8-byte entries is one LOP3); index = count below + (y >
                            // boundary in the cell), a tie staying below, as with the 256-cell grid
                            static_assert(kWideCopies * 8 == 32, "the cell bits give the entry group's byte offset");
                            const float u = __saturatef(fmaf(yv[e2], wide_s, 0.5f));
                            const float g = fmaf(u, 1023.75f, 393216.0f);
                            const uint2 ent = lds_u64(wide_lane + (__float_as_uint(g) & ((kWideCells - 1u) << 5)));
                            const uint32_t diff = __float_as_uint(__fsub_rn(__uint_as_float(ent.x), yv[e2]));
                            add_field<BITS>(w, 2 * j2 + e2, __umulhi(diff, 2u) + ent.y);
                            continue;
                        }
                        const uint32_t cb = cell[e2] & static_cast<uint32_t>((C::kLutEntries - 1) << 7);
                        const uint32_t e = lds_u32(Lo::kAlignLut ? (cb | lut_lane) : (lut_lane + cb));
                        // the entry read as a float is the cell's boundary moved by at most 15 ulps (its low 4 bits
                        // hold the count; the boundary's own low bits are zero), or +inf / a NaN when it has none.
                        // The sign of (boundary - y) is set exactly when y lies above the boundary (ties stay below);
                        // +inf - y is +inf and NaN - y the canonical, positive NaN.
                        // index = count + (sign bit of the difference): the high word of diff * 2 is that bit,
                        // so one multiply-high with the count as addend gives the index
                        const uint32_t diff = __float_as_uint(__fsub_rn(__uint_as_float(e), yv[e2]));
                        add_field<BITS>(w, 2 * j2 + e2, __umulhi(diff, 2u) + (e & 15u));
                    }
                }
                const int boff = (c0 + k * 32) * BITS / 8;
                if (staged) {
#pragma unroll
                    for (int i = 0; i < BITS; ++i) reinterpret_cast<uint32_t*>(pk + boff)[i] = w[i];
                } else if (orow >= 0) {
                    store_words<BITS>(packed + orow * kRowBytes + boff, w);
                }
            }
            if constexpr (SLOTS) {
                if (c0 == 0 && orow >= 0) norms[orow] = s_norm[s * 128 + r].x;
                __syncwarp();
                if (lane == 0) mbar_arrive(b_nfree + 8 * s);
            }
            if (staged) {
                // make this warp's rows visible to the bulk copy engine, then hand the tile to the issuer
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_pkfull + 8 * pb);
                if (issuer) {
                    if (!mbar_wait(b_pkfull + 8 * pb, (li >> 1) & 1, abort_flag, wait_limit)) break;
                    const int64_t rows = (n - tile * 128 < 128) ? n - tile * 128 : 128;
                    const uint32_t bytes = static_cast<uint32_t>(rows * kRowBytes);
                    const uint32_t bulk = bytes & ~15u;
                    uint8_t* gdst = packed + tile * 128 * kRowBytes;
                    const uint32_t ssrc = smem_u32(s_pk + pb * Lo::kPkBytes);
                    if (bulk) bulk_store(gdst, ssrc, bulk);
                    for (uint32_t o = bulk; o < bytes; o += 4)       // a ragged tail of whole words
                        *reinterpret_cast<uint32_t*>(gdst + o) =
                            *reinterpret_cast<const uint32_t*>(s_pk + pb * Lo::kPkBytes + o);
                    bulk_commit();
                    bulk_wait_read<1>();                          // the previous tile's buffer has been read
                    if (li >= 1) mbar_arrive(b_pkempty + 8 * (pb ^ 1));
                }
            }
        }
        if (staged && issuer) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// Decode CTA: warp 0 producer, warp 1 TMEM owner + MMA issuer, warps 2.. builders/epilogue (kEpiWarps:
// warp w works on rows 32*(w%4).. and owns kCols columns of them).
template <int D>
struct DecCfg {
    static constexpr int kEpiWarps = (D == 128) ? 16 : 8;
    static constexpr int kThreads = 32 * (2 + kEpiWarps);
    static constexpr int kCols = D * 4 / kEpiWarps;          // 32, 32, 128
    static constexpr int kChunks = kCols / 32;
};

template <int D, int BITS>
struct DecLayout {
    using C = KeyCfg<D>;
    using E = DecCfg<D>;
    static constexpr int kRowBytes = D * BITS / 8;
    static constexpr int kInBytes = 128 * kRowBytes + 128 * 4;            // packed rows + norms
    // staging buffers for the packed rows: the producer runs up to kInBufs - 1 tiles ahead of the builders
    // (a buffer is released once its tile's A values are stored; measured best: 6 up to 3 bits, else 4)
    static constexpr int kInBufs = (D == 256) ? 1 : (BITS <= 3 ? 6 : 4);
    // code-pair table: one copy per shared-memory bank (entry e of lane l at 128 e + 4 l) where it fits
    static constexpr bool kReplPairs = (D <= 128);
    // up to 4 bits the table maps a pair of codes to a half2 of levels; from 5 bits (2^(2 bits) pairs would not
    // fit) it maps one code to its fp16 level (low half) and a half2 takes two lookups
    static constexpr int kEntries = (BITS > 4) ? (1 << BITS) : (1 << (2 * BITS));
    static constexpr int kPairBytes = kEntries * (kReplPairs ? 128 : 4);
    // d <= 128: the A tile (the looked-up codebook values) is built in tensor memory with tcgen05.st and the MMA
    // reads it from there, which takes its writes and the tensor core's reads off shared memory; d = 256 keeps
    // it in shared memory (its two accumulators fill the 512 TMEM columns)
    static constexpr bool kTmemA = (D <= 128);
    static constexpr uint32_t kTmemCols = kTmemA ? (D == 128 ? 512 : 256) : C::kTmemCols;
    static constexpr uint32_t kTmemACol = 2 * D;                              // A buffer b at 2 D + b D / 2
    static constexpr uint32_t kPit = 0;
    static constexpr uint32_t kA = kPit + C::kPiBytes;
    static constexpr uint32_t kIn = kA + (kTmemA ? 0 : C::kDecBufs * C::kTileBytes);
    static constexpr uint32_t kPair = kIn + kInBufs * kInBytes;
    // where the slack fits, the replicated table is placed on a multiple of its size, so a lookup address is
    // (pair bits << 7) | lane bits: one funnel shift and one LOP3 per lookup
    static constexpr int kPatchBufs = (D <= 128) ? 2 : 1;
    static constexpr uint32_t kPatchBytes = 32 * 64;
    static constexpr int kBars = 2 * C::kDecBufs + 2 * kInBufs + 8;
    static constexpr uint32_t kTailBytes = E::kEpiWarps * kPatchBufs * kPatchBytes + 8 * kBars + 16 + 1024;
    static constexpr bool kAlignPairs = kReplPairs && BITS <= 4 &&
        (((kPair + 2 * kPairBytes + 511) & ~511u) + kTailBytes <= 227 * 1024);
    static constexpr uint32_t kPairRegion = kAlignPairs ? 2 * kPairBytes : kPairBytes;
    // per-warp output patches: 32 rows x 64 bytes, 64B-swizzled, the source of one tensor store each
    static constexpr uint32_t kPatch = (kPair + kPairRegion + 511) & ~511u;    // 64B swizzle repeats every 512 bytes
    static constexpr uint32_t kBar = kPatch + E::kEpiWarps * kPatchBufs * kPatchBytes;
    static constexpr uint32_t kMisc = kBar + 8 * kBars;
    static constexpr uint32_t kBytes = kMisc + 16 + 1024;
    static_assert(kBytes <= 227 * 1024, "decode layout exceeds the shared memory of one CTA");
};

template <int D, int BITS>
__host__ __device__ constexpr uint32_t dec_smem_bytes() {
    return DecLayout<D, BITS>::kBytes;
}

template <int D, int BITS, bool OUT_F32>
__global__ void __launch_bounds__(DecCfg<D>::kThreads, 1)
    decode_k_kernel(const __grid_constant__ CUtensorMap tmap_pit, const __grid_constant__ CUtensorMap tmap_out,
                    const uint32_t* __restrict__ pair_lut_g, const uint8_t* __restrict__ packed,
                    const float* __restrict__ norms, int64_t n) {
    using C = KeyCfg<D>;
    using E = DecCfg<D>;
    using Lo = DecLayout<D, BITS>;
    constexpr int NB = C::kDecBufs;
    constexpr int NI = Lo::kInBufs;
    constexpr int kRowBytes = Lo::kRowBytes;
    constexpr int kPartWords = E::kCols * BITS / 32;   // 32-bit words of this warp's columns of a packed row
    constexpr int kPairs = Lo::kEntries;
    constexpr int kOutBytes = OUT_F32 ? 4 : 2;
    constexpr int kPasses = 32 * kOutBytes / 64;   // 64-byte row segments of one 32-column chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);   // stays a shared-space pointer
    uint8_t* s_pit = smem + Lo::kPit;
    uint8_t* s_a = smem + Lo::kA;
    uint8_t* s_in = smem + Lo::kIn;
    const uint32_t pair_base = Lo::kAlignPairs
        ? (smem_u32(smem + Lo::kPair) + Lo::kPairBytes - 1) & ~static_cast<uint32_t>(Lo::kPairBytes - 1)
        : smem_u32(smem + Lo::kPair);
    uint32_t* s_pair = reinterpret_cast<uint32_t*>(smem + (pair_base - smem_u32(smem)));
    const uint32_t bar0 = smem_u32(smem + Lo::kBar);
    const uint32_t b_afull = bar0, b_aempty = b_afull + 8 * NB, b_infull = b_aempty + 8 * NB,
                   b_inempty = b_infull + 8 * NI, b_accfull = b_inempty + 8 * NI, b_accempty = b_accfull + 16,
                   b_pifull = b_accempty + 16, b_final = b_pifull + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lo::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t num_tiles = (n + 127) / 128;

    if (threadIdx.x == 0) {
        for (int b = 0; b < NB; ++b) {
            mbar_init(b_afull + 8 * b, E::kEpiWarps);
            mbar_init(b_aempty + 8 * b, 1);
        }
        for (int b = 0; b < NI; ++b) {
            mbar_init(b_infull + 8 * b, 1);
            mbar_init(b_inempty + 8 * b, E::kEpiWarps);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(b_accfull + 8 * a, 1);
            mbar_init(b_accempty + 8 * a, E::kEpiWarps);
        }
        mbar_init(b_pifull, 1);
        mbar_init(b_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Lo::kTmemCols);
        tmem_relinquish();
    }
    if constexpr (Lo::kReplPairs) {
        fill_replicated(s_pair, pair_lut_g, kPairs);
    } else {
        for (int i = threadIdx.x; i < kPairs; i += blockDim.x) s_pair[i] = pair_lut_g[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // a tile's packed rows and norms go through the staging buffer when both copies are 16-byte multiples
    auto tile_rows = [&](int64_t tile) -> int64_t { return (n - tile * 128 < 128) ? n - tile * 128 : 128; };
    auto bulk_ok = [&](int64_t rows) -> bool { return ((rows * kRowBytes) % 16 == 0) && ((rows * 4) % 16 == 0); };
    // 0 at run time (the host rejects n < 0) but unknown to the compiler: ties a load to a later use (below)
    const uint32_t opaque_zero = static_cast<uint32_t>(static_cast<uint64_t>(n) >> 63);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            mbar_arrive_expect_tx(b_pifull, C::kPiBytes);
            for (int kb = 0; kb < C::kKB; ++kb)
                tma_load_2d(smem_u32(s_pit + kb * C::kPiBlockBytes), &tmap_pit, b_pifull, kb * 64, 0);
            int li = 0;
            for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++li) {
                const int ib = li % NI;
                if (!mbar_wait(b_inempty + 8 * ib, ((li / NI) & 1) ^ 1, abort_flag)) break;
                const int64_t rows = tile_rows(tile);
                if (bulk_ok(rows)) {
                    const uint32_t pb = static_cast<uint32_t>(rows * kRowBytes), nbytes = static_cast<uint32_t>(rows * 4);
                    mbar_arrive_expect_tx(b_infull + 8 * ib, pb + nbytes);
                    uint8_t* dst = s_in + ib * Lo::kInBytes;
                    bulk_load(smem_u32(dst), packed + tile * 128 * kRowBytes, pb, b_infull + 8 * ib);
                    bulk_load(smem_u32(dst + 128 * kRowBytes), norms + tile * 128, nbytes, b_infull + 8 * ib);
                } else {
                    mbar_arrive(b_infull + 8 * ib);              // ragged tail: read straight from global
                }
            }
            for (int k = (li > NI ? li - NI : 0); k < li; ++k) mbar_wait_drain(b_infull + 8 * (k % NI), (k / NI) & 1);
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
                const uint32_t pa = smem_u32(s_pit);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k & 3) * 32;
                    const uint64_t bd = desc_kmajor_sw128(pa + (k >> 2) * C::kPiBlockBytes + off);
                    if constexpr (Lo::kTmemA) {
                        umma_f16_ts(d_tmem, tmem_base + Lo::kTmemACol + b * (D / 2) + 8 * k, bd, C::kIdesc, k > 0 ? 1u : 0u);
                    } else {
                        const uint32_t aa = smem_u32(s_a + b * C::kTileBytes);
                        const uint64_t ad = desc_kmajor_sw128(aa + (k >> 2) * C::kTileBlockBytes + off);
                        umma_f16_ss(d_tmem, ad, bd, C::kIdesc, k > 0 ? 1u : 0u);
                    }
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
        const int c0 = (ew >> 2) * E::kCols;               // first column of this warp
        const int r = quarter * 32 + lane;
        uint8_t* patches = smem + Lo::kPatch + ew * Lo::kPatchBufs * Lo::kPatchBytes;
        const uint32_t pair_lane = pair_base + 4u * lane;          // this lane's copy of the pair table
        int pcount = 0;                                    // tensor stores issued by this warp
        float nrm_next = 0.f;

        // build the A tile (c_op[idx] as fp16: TMEM rows, or 128B-swizzled K-major smem) for local tile index lt
        auto build = [&](int lt, int64_t tile) -> bool {
            const int b = lt % NB, ib = lt % NI;
            if (!mbar_wait(b_aempty + 8 * b, ((lt / NB) & 1) ^ 1, abort_flag)) return false;
            if (!mbar_wait(b_infull + 8 * ib, (lt / NI) & 1, abort_flag)) return false;
            const int64_t rows = tile_rows(tile);
            const int64_t row = tile * 128 + r;
            uint32_t w[kPartWords + 1];
            w[kPartWords] = 0u;
            if (r < rows) {
                auto& wp = *reinterpret_cast<uint32_t(*)[kPartWords]>(w);
                if (bulk_ok(rows)) {
                    nrm_next = reinterpret_cast<const float*>(s_in + ib * Lo::kInBytes + 128 * kRowBytes)[r];
                    load_words<kPartWords>(s_in + ib * Lo::kInBytes + r * kRowBytes + c0 * BITS / 8, wp);
                    // the norm is used only a tile later: make the lookups (and so the A store that precedes the
                    // release of this buffer) depend on its load as well
                    w[0] |= __float_as_uint(nrm_next) & opaque_zero;
                } else {
                    nrm_next = norms[row];
                    load_words<kPartWords>(packed + row * kRowBytes + c0 * BITS / 8, wp);   // ragged tail
                }
            } else {
#pragma unroll
                for (int i = 0; i < kPartWords; ++i) w[i] = 0u;
                nrm_next = 0.f;
            }
            // one half2 of codebook values per code pair (two consecutive columns of the row)
            auto pair_value = [&](int c, int p) -> uint32_t {
                if constexpr (BITS > 4) {
                    // two single-code lookups, merged into one half2 (first column in the low half)
                    const uint32_t i0 = get_bits<BITS>(w, (c * 8 + 2 * p) * BITS);
                    const uint32_t i1 = get_bits<BITS>(w, (c * 8 + 2 * p + 1) * BITS);
                    const uint32_t v0 = Lo::kReplPairs ? lds_u32(pair_lane + i0 * 128u) : s_pair[i0];
                    const uint32_t v1 = Lo::kReplPairs ? lds_u32(pair_lane + i1 * 128u) : s_pair[i1];
                    return __byte_perm(v0, v1, 0x5410);
                } else if constexpr (Lo::kAlignPairs) {
                    const uint32_t x = bits_shr(w, (c * 8 + 2 * p) * BITS - 7);
                    return lds_u32((x & (static_cast<uint32_t>(kPairs - 1) << 7)) | pair_lane);
                } else {
                    const uint32_t key = get_bits<2 * BITS>(w, (c * 8 + 2 * p) * BITS);
                    return Lo::kReplPairs ? lds_u32(pair_lane + key * 128u) : s_pair[key];
                }
            };
            if constexpr (Lo::kTmemA) {
                static_assert(E::kCols == 32, "one 16-column TMEM store per warp and tile");
                // the MMA that last read this A buffer has completed (aempty): order the stores after it
                tc_fence_after();
                uint32_t hc[16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int p = 0; p < 4; ++p) hc[4 * c + p] = pair_value(c, p);
                }
                tmem_st_32x32b_x16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + Lo::kTmemACol +
                                       b * (D / 2) + c0 / 2,
                                   hc);
                tmem_st_wait();
                tc_fence_before();
            } else {
                uint8_t* as = s_a + b * C::kTileBytes;
#pragma unroll
                for (int c = 0; c < E::kCols / 8; ++c) {
                    uint32_t h[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) h[p] = pair_value(c, p);
                    const int col = c0 + c * 8;
                    *reinterpret_cast<uint4*>(as + (col >> 6) * C::kTileBlockBytes + sw128_offset(r, (col & 63) >> 3)) =
                        make_uint4(h[0], h[1], h[2], h[3]);
                }
                fence_proxy_async_smem();
            }
            // The staging buffer is released only now: the A values just stored were looked up from every word
            // (and the norm) this warp read from it, so those reads have completed. Releasing it straight after
            // issuing the loads let the next bulk copy into the buffer overwrite words that a bank-conflicted
            // shared load (128-byte rows at 8 bits: all 32 lanes in one bank) was still reading.
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(b_inempty + 8 * ib);
                mbar_arrive(b_afull + 8 * b);
            }
            return true;
        };

        bool ok = true;
        int64_t tile = blockIdx.x;
        if (tile < num_tiles) ok = build(0, tile);
        int li = 0;
        for (; ok && tile < num_tiles; tile += gridDim.x, ++li) {
            const float nrm = nrm_next;
            const int64_t next = tile + gridDim.x;
            if (next < num_tiles && !build(li + 1, next)) break;
            const int a = li & 1;
            if (!mbar_wait(b_accfull + 8 * a, (li >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * D + c0;
#pragma unroll
            for (int ch = 0; ch < E::kChunks; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + ch * 32, v);
                tmem_ld_wait();
                if (ch == E::kChunks - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b_accempty + 8 * a);
                }
                // per 64-byte segment of this row's chunk: scale, convert and write it as row r of the warp's
                // 64B-swizzled patch (32 rows x 64 bytes); one lane then stores the patch with a tensor store
                // (rows past n are clipped by the tensor map)
                const int col0 = c0 + ch * 32;
#pragma unroll
                for (int ps = 0; ps < kPasses; ++ps) {
                    uint8_t* patch = patches + (pcount % Lo::kPatchBufs) * Lo::kPatchBytes;
                    if (pcount >= Lo::kPatchBufs) {
                        // the store that last read this patch is done reading it
                        if (lane == 0) {
                            if constexpr (Lo::kPatchBufs == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();
                        }
                        __syncwarp();
                    }
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc) {
                        uint4 pk;
                        if constexpr (OUT_F32) {
                            const int e0 = (ps * 4 + pc) * 4;
                            pk = make_uint4(__float_as_uint(__uint_as_float(v[e0]) * nrm),
                                            __float_as_uint(__uint_as_float(v[e0 + 1]) * nrm),
                                            __float_as_uint(__uint_as_float(v[e0 + 2]) * nrm),
                                            __float_as_uint(__uint_as_float(v[e0 + 3]) * nrm));
                        } else {
                            uint32_t hw[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                // two elements per packed f32x2 multiply, then one paired conversion
                                const float2 y2 = __fmul2_rn(make_float2(__uint_as_float(v[8 * pc + 2 * k]),
                                                                         __uint_as_float(v[8 * pc + 2 * k + 1])),
                                                             make_float2(nrm, nrm));
                                __half2 h2 = __floats2half2_rn(y2.x, y2.y);
                                hw[k] = *reinterpret_cast<uint32_t*>(&h2);
                            }
                            pk = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        }
                        *reinterpret_cast<uint4*>(patch + lane * 64 + ((pc ^ ((lane >> 1) & 3)) * 16)) = pk;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmap_out, smem_u32(patch), col0 + ps * (64 / kOutBytes),
                                     static_cast<int>(tile * 128 + quarter * 32));
                        bulk_commit();
                    }
                    ++pcount;
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Lo::kTmemCols);
    }
}

}  // namespace dev
}  // namespace tq
