// QJL residual keys: the second stage of a QJL key code.
//
// "KV Cache API" (TurboQuant docs), compressors.py TurboQuantCompressorV2.compress: a key is first coded by the
// MSE compressor at bits - 1 (norm, rotation, nearest codebook level); the residual r = x - k_mse of that
// reconstruction is then sketched by one sign bit per row of a seeded Gaussian matrix S, sign(S r), and its
// norm ||r|| is kept.  asymmetric_attention_scores estimates <q, k> as <q, k_mse> + ||r|| sqrt(pi/2) / m
// <S q, signs>, m the rows of S.
//
// This kernel takes the MSE stage (packed indices and norms, written by the key encoder) and the fp16 rows, and
// writes the sign bits and ||r||:
//   k_mse = n * Pi_op^T c_op[idx]            (tensor cores: fp16 codebook pairs x fp16 Pi_op, f32 accumulate)
//   r     = x - k_mse                        (f32)
//   rho   = ||r||                            (f32)
//   sign  = (S_op r >= 0)                    (tensor cores: fp16 hi + lo halves of r x fp16 S_op, f32 accumulate)
// One warp owns 16 rows; the products are mma.sync m16n8k16 tiles (the residual needs an exact f32 subtraction
// between the two products, and the kernel is not on the decode step's path).
#pragma once

#include "tq_device.cuh"

namespace tq {
namespace dev {

// Warps per CTA: 4 at d <= 128, 2 at d = 256 (its matrix tile takes 135 KB of shared memory).
template <int D>
__host__ __device__ constexpr int qjl_warps() { return D == 256 ? 2 : 4; }

// S is drawn from the generator seeded with the codec's seed plus this offset (compressors.py seeds the sketch
// with seed + 10000)
constexpr uint64_t kQjlSeedOffset = 10000;

template <int D>
__host__ __device__ constexpr int qjl_r_stride() { return D + 8; }     // f32 residual row in shared memory, padded

template <int D>
__host__ __device__ constexpr int qjl_m_stride() { return D + 8; }     // fp16 matrix row in shared memory, padded

template <int D, int KB>
__host__ __device__ constexpr int qjl_smem_bytes() {
    return D * qjl_m_stride<D>() * 2 +                                   // Pi_op^T, then S_op
           (1 << (2 * KB)) * 128 +                                       // replicated code-pair table
           qjl_warps<D>() * 16 * (D * KB / 32 + 1) * 4 +                 // packed index rows
           qjl_warps<D>() * 16 * qjl_r_stride<D>() * 4;                  // residual rows
}

__device__ __forceinline__ void qjl_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t qjl_pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// fp16 hi + lo halves of a pair of floats: hi = fp16(x), lo = fp16(x - hi); hi + lo is within 2^-22 |x| of x
// while x - hi stays in fp16's normal range.
__device__ __forceinline__ void qjl_split(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 hf = __half22float2(h);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = qjl_pack_f16(x0 - hf.x, x1 - hf.y);
}

// A d x d fp16 matrix (row-major in global memory) into shared memory with rows padded to qjl_m_stride<D>()
// halves, so that the eight rows x four column pairs of one B-fragment load fall in 32 distinct banks.
template <int D>
__device__ __forceinline__ void qjl_stage_matrix(__half* dst, const __half* __restrict__ src) {
    constexpr int kVec = D / 8;                                       // uint4 per row
    for (int i = threadIdx.x; i < D * kVec; i += blockDim.x) {
        const int r = i / kVec, c = i % kVec;
        *reinterpret_cast<uint4*>(dst + r * qjl_m_stride<D>() + 8 * c) =
            __ldg(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r) * D) + c);
    }
}

// grid: ceil(n / (16 qjl_warps)) CTAs; warp w of CTA c owns input rows 16 (qjl_warps c + w) .. + 15.
// Input row i is x[i * x_stride ..]; its codes, norm, signs and rho live at pool row slots[i] (i without a slot
// mapping; a negative slot skips the row).  pi_t = Pi_op^T row-major (pi_t[i][j] = Pi_op[j][i]); s_op row-major.
// Both products read their B operand from a padded copy of the matrix in shared memory: first Pi_op^T, then S_op.
template <int D, int KB>
__global__ void __launch_bounds__(32 * qjl_warps<D>()) qjl_residual_kernel(
    const __half* __restrict__ x, int64_t n, int64_t x_stride, const int64_t* __restrict__ slots,
    const uint8_t* __restrict__ packed, const float* __restrict__ norms, const uint32_t* __restrict__ pair_lut,
    const __half* __restrict__ pi_t, const __half* __restrict__ s_op, uint8_t* __restrict__ signs,
    float* __restrict__ rho) {
    constexpr int W = qjl_warps<D>();
    constexpr int KROW = D * KB / 8;                // bytes of one packed index row
    constexpr int KW = KROW / 4;                    // 32-bit words of it (D * KB is a multiple of 32)
    constexpr int KS = D / 16;                      // k-steps over the d coordinates
    constexpr int NTB = 8;                          // n-tiles (64 output columns) per pass
    constexpr int NPASS = D / (8 * NTB);
    constexpr int RS = qjl_r_stride<D>();
    constexpr int MS = qjl_m_stride<D>();
    constexpr int kPairs = 1 << (2 * KB);
    extern __shared__ __align__(16) uint8_t smem[];
    __half* s_mat = reinterpret_cast<__half*>(smem);
    uint32_t* s_lut = reinterpret_cast<uint32_t*>(smem + D * MS * 2);
    uint32_t* s_codes = s_lut + kPairs * 32;
    float* s_r = reinterpret_cast<float*>(s_codes + W * 16 * (KW + 1));
    qjl_stage_matrix<D>(s_mat, pi_t);
    fill_replicated(s_lut, pair_lut, kPairs);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * W + warp) * 16;
    const bool active = row0 < n;                   // warps past the rows still take part in the CTA barriers
    uint32_t* codes = s_codes + warp * 16 * (KW + 1);
    float* rr = s_r + warp * 16 * RS;

    // pool rows and norms of this lane's rows gid and gid + 8 (-1: no row)
    int64_t prow[2];
    float nrm[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t i = row0 + gid + 8 * h;
        prow[h] = (i < n) ? (slots ? slots[i] : i) : -1;
        nrm[h] = (prow[h] >= 0) ? norms[prow[h]] : 0.f;
    }
    // the warp's 16 packed index rows, word by word, plus one zero word of padding per row (zero for missing rows)
    for (int i = lane; i < 16 * (KW + 1); i += 32) {
        const int r = i / (KW + 1), wv = i % (KW + 1);
        const int64_t gi = row0 + r;
        uint32_t v = 0;
        if (gi < n && wv < KW) {
            const int64_t pr = slots ? slots[gi] : gi;
            if (pr >= 0) v = __ldg(reinterpret_cast<const uint32_t*>(packed + pr * KROW) + wv);
        }
        codes[i] = v;
    }
    __syncthreads();                                // matrix, table and index rows in place
    const uint32_t lane_addr = smem_u32(s_lut) + 4u * lane;
    // code pair of row r starting at coordinate c (c even): 2 KB bits of the row's LSB-first bitstream
    auto pair_of = [&](int r, int c) -> uint32_t {
        const int bit = c * KB, wi = bit >> 5, sh = bit & 31;
        const uint32_t* w = codes + r * (KW + 1);
        const uint32_t v = sh ? __funnelshift_r(w[wi], w[wi + 1], sh) : w[wi];
        return lds_u32(lane_addr + ((v & (kPairs - 1)) << 7));
    };

    // ---- k_mse = n * Pi_op^T c_op[idx], r = x - k_mse, ||r||^2; 64 columns per pass
    float ss[2] = {0.f, 0.f};
    if (active) {
        for (int pass = 0; pass < NPASS; ++pass) {
            float acc[NTB][4];
#pragma unroll
            for (int t = 0; t < NTB; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
            for (int ks = 0; ks < KS; ++ks) {
                const int c0 = 16 * ks + 2 * tig;
                const uint32_t a0 = pair_of(gid, c0), a1 = pair_of(gid + 8, c0);
                const uint32_t a2 = pair_of(gid, c0 + 8), a3 = pair_of(gid + 8, c0 + 8);
#pragma unroll
                for (int t = 0; t < NTB; ++t) {
                    const __half* bp = s_mat + (8 * (pass * NTB + t) + gid) * MS + c0;
                    qjl_mma(acc[t], a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(bp),
                            *reinterpret_cast<const uint32_t*>(bp + 8));
                }
            }
#pragma unroll
            for (int t = 0; t < NTB; ++t) {
                const int col = 8 * (pass * NTB + t) + 2 * tig;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t i = row0 + gid + 8 * h;
                    float2 xv = make_float2(0.f, 0.f);
                    if (prow[h] >= 0) xv = __half22float2(*reinterpret_cast<const __half2*>(x + i * x_stride + col));
                    const float r0 = (prow[h] >= 0) ? xv.x - nrm[h] * acc[t][2 * h] : 0.f;
                    const float r1 = (prow[h] >= 0) ? xv.y - nrm[h] * acc[t][2 * h + 1] : 0.f;
                    ss[h] = fmaf(r0, r0, fmaf(r1, r1, ss[h]));
                    *reinterpret_cast<float2*>(rr + (gid + 8 * h) * RS + col) = make_float2(r0, r1);
                }
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            ss[h] += __shfl_xor_sync(0xffffffffu, ss[h], 1);
            ss[h] += __shfl_xor_sync(0xffffffffu, ss[h], 2);
            if (tig == 0 && prow[h] >= 0) rho[prow[h]] = sqrtf(ss[h]);
        }
    }
    __syncthreads();                                // every warp is done with Pi_op^T
    qjl_stage_matrix<D>(s_mat, s_op);
    __syncthreads();
    if (!active) return;

    // ---- proj = S_op r with r as fp16 hi + lo halves; sign bits LSB-first, byte t = columns 8 t .. 8 t + 7
    for (int pass = 0; pass < NPASS; ++pass) {
        float acc[NTB][4];
#pragma unroll
        for (int t = 0; t < NTB; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
        for (int ks = 0; ks < KS; ++ks) {
            const int c0 = 16 * ks + 2 * tig;
            uint32_t ah[4], al[4];
            const float2 v0 = *reinterpret_cast<const float2*>(rr + gid * RS + c0);
            const float2 v1 = *reinterpret_cast<const float2*>(rr + (gid + 8) * RS + c0);
            const float2 v2 = *reinterpret_cast<const float2*>(rr + gid * RS + c0 + 8);
            const float2 v3 = *reinterpret_cast<const float2*>(rr + (gid + 8) * RS + c0 + 8);
            qjl_split(v0.x, v0.y, ah[0], al[0]);
            qjl_split(v1.x, v1.y, ah[1], al[1]);
            qjl_split(v2.x, v2.y, ah[2], al[2]);
            qjl_split(v3.x, v3.y, ah[3], al[3]);
#pragma unroll
            for (int t = 0; t < NTB; ++t) {
                const __half* bp = s_mat + (8 * (pass * NTB + t) + gid) * MS + c0;
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(bp);
                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(bp + 8);
                qjl_mma(acc[t], ah[0], ah[1], ah[2], ah[3], b0, b1);
                qjl_mma(acc[t], al[0], al[1], al[2], al[3], b0, b1);
            }
        }
#pragma unroll
        for (int t = 0; t < NTB; ++t) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t byte = ((acc[t][2 * h] >= 0.f) ? 1u : 0u) << (2 * tig);
                byte |= ((acc[t][2 * h + 1] >= 0.f) ? 1u : 0u) << (2 * tig + 1);
                byte |= __shfl_xor_sync(0xffffffffu, byte, 1);
                byte |= __shfl_xor_sync(0xffffffffu, byte, 2);
                if (tig == 0 && prow[h] >= 0) signs[prow[h] * (D / 8) + pass * NTB + t] = static_cast<uint8_t>(byte);
            }
        }
    }
}

}  // namespace dev
}  // namespace tq
