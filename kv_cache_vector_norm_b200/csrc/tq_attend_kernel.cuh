// Fused decode-step attention over the compressed cache.
//
// "KV Cache API" (TurboQuant docs), store.py TurboQuantKVCache.attention_scores / attend: logits
// q . k * scale (scale 1/sqrt(head_dim) by default), softmax, weights @ dequantised values; the page
// materialises fp32 keys and values to do it.  "turbo-attn": the decode kernel is split-K over the paged
// cache and rotates the query once, so scores need no un-rotation.  Here neither keys nor values are
// ever materialised:
//   score_t = scale * n_t * <Pi_op q, c_op[idx_t]>       (tensor cores: fp16 codebook values x fp16
//                                                         hi/lo halves of the rotated query)
//   out     = sum_t p_t (q_t s_t + z_t) / sum_t p_t       (tensor cores: integer codes x bf16 hi/lo
//                                                         halves of p_t s_t; the zero term on FMAs)
// One CTA = one (split, kv head, sequence); warp 4 streams 16-token chunks of every pool array into a
// shared-memory ring with bulk TMA copies; warps 0..3 each consume one chunk of every stage with
// mma.sync fragments kept in registers; the last CTA of a (sequence, kv head) merges the splits.
#pragma once

#include "tq_device.cuh"

namespace tq {
namespace dev {

struct AttendParams {
    int batch, num_q_heads, num_kv_heads, group;     // group = H_q / H_kv (<= 8)
    float scale_log2;                                // softmax scale * log2(e)
    int64_t max_seq_len;
    const int32_t* block_table;                      // NULL: contiguous layout
    int max_blocks;
    const int32_t* seq_lens;                         // nullable (contiguous)
    const __half* q;
    const __half* pi_op;                             // d x d row-major
    const uint32_t* pair_lut;                        // 2^(2 kb) half2 pairs of codebook values
    const uint8_t* k_packed;
    const float* k_norms;
    const uint8_t* v_data;
    const __half* v_scales;
    const __half* v_zeros;
    float* out;
    float* partials;                                 // [B][H_kv][splits][16 + 8 d]
    int* counters;                                   // [B][H_kv]
    int num_splits;
};

template <int D, int KB, int VB, int VG>
struct AttCfg {
    static constexpr int kWarps = 4;                 // consumer warps
    static constexpr int kThreads = 32 * (kWarps + 1);
    static constexpr int kChunkTok = 16;             // tokens per chunk (= one paged block)
    static constexpr int kStages = 4;
    static constexpr int kKRow = D * KB / 8;
    static constexpr int kVRow = D * VB / 8;
    static constexpr int kVGroups = D / VG;
    static constexpr int kKOff = 0;
    static constexpr int kNOff = kKOff + kChunkTok * kKRow;
    static constexpr int kVOff = kNOff + kChunkTok * 4;
    static constexpr int kSOff = kVOff + kChunkTok * kVRow;
    static constexpr int kZOff = kSOff + kChunkTok * kVGroups * 2;
    static constexpr int kChunkBytes = kZOff + kChunkTok * kVGroups * 2;
    static constexpr int kStageBytes = kWarps * kChunkBytes;
    static constexpr int kQuarterBits = D * KB / 4;  // one lane's quarter of a key row (16-bit multiple)
    static constexpr int kQuarterHalves = kQuarterBits / 16;
    static constexpr int kQuarterWords = (kQuarterHalves + 1) / 2 + 1;
    static constexpr int kMinBlocks = (D == 256) ? 1 : 3;
    static constexpr int kPartFloats = 16 + 8 * D;
    // shared memory: stages | q fragments | rotated q | pair lut | reduction | barriers
    static constexpr int kCombineFloats = kWarps * kPartFloats;
    static constexpr int kRingBytes =
        (kStages * kStageBytes > kCombineFloats * 4) ? kStages * kStageBytes : kCombineFloats * 4;
    static constexpr int kQfOff = kRingBytes;
    static constexpr int kQrOff = kQfOff + (D / 16) * 32 * 16;
    static constexpr int kLutOff = kQrOff + 8 * D * 4;
    static constexpr int kRedOff = kLutOff + (1 << (2 * KB)) * 4;
    static constexpr int kBarOff = (kRedOff + 8 * 4 + 15) & ~15;
    static constexpr int kSmem = kBarOff + 8 * (2 * kStages) + 16;
    static_assert(kChunkBytes % 16 == 0 && kNOff % 16 == 0 && kVOff % 16 == 0 && kSOff % 16 == 0 && kZOff % 16 == 0,
                  "bulk copies need 16-byte multiples");
};

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint4& a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint4& a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// hi/lo bf16 split of two values: hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16(x0, x1);
    const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
    lo = pack_bf16(x0 - h0, x1 - h1);
}

// bf16x2 {code[token a][col], code[token b][col]} of the value codes (exact small integers).
template <int VB>
__device__ __forceinline__ uint32_t vcode_pair(const uint8_t* row_a, const uint8_t* row_b, int col) {
    if constexpr (VB == 2 || VB == 4) {
        const int bit = col * VB;
        const uint32_t wa = *reinterpret_cast<const uint32_t*>(row_a + (bit >> 5) * 4);
        const uint32_t wb = *reinterpret_cast<const uint32_t*>(row_b + (bit >> 5) * 4);
        const int sh = bit & 31;
        // put the 16-bit halves holding the field side by side, then mask into a bf16 magic of 128
        const uint32_t z = (sh < 16) ? __byte_perm(wa, wb, 0x5410) : __byte_perm(wa, wb, 0x7632);
        const uint32_t m = (VB == 2) ? 0x00030003u : 0x000F000Fu;
        const uint32_t v = ((z >> (sh & 15)) & m) | 0x43004300u;
        __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v), __floats2bfloat162_rn(128.f, 128.f));
        return *reinterpret_cast<uint32_t*>(&r);
    } else if constexpr (VB == 8) {
        return pack_bf16(static_cast<float>(row_a[col]), static_cast<float>(row_b[col]));
    } else {
        const int bit = col * VB, byte = bit >> 3, sh = bit & 7;
        uint32_t qa = row_a[byte], qb = row_b[byte];
        if (sh + VB > 8) {
            qa |= static_cast<uint32_t>(row_a[byte + 1]) << 8;
            qb |= static_cast<uint32_t>(row_b[byte + 1]) << 8;
        }
        qa = (qa >> sh) & ((1u << VB) - 1u);
        qb = (qb >> sh) & ((1u << VB) - 1u);
        return pack_bf16(static_cast<float>(qa), static_cast<float>(qb));
    }
}

template <int D, int KB, int VB, int VG>
__global__ void __launch_bounds__(AttCfg<D, KB, VB, VG>::kThreads, AttCfg<D, KB, VB, VG>::kMinBlocks)
    attend_kernel(const AttendParams p) {
    using C = AttCfg<D, KB, VB, VG>;
    constexpr int S = C::kStages;
    constexpr int KS = D / 16;                        // k-steps of the score contraction
    constexpr int NT = D / 8;                         // n-tiles of the value contraction
    constexpr int G8 = C::kVGroups;
    extern __shared__ __align__(16) uint8_t smem[];
    uint4* s_qf = reinterpret_cast<uint4*>(smem + C::kQfOff);
    float* s_qr = reinterpret_cast<float*>(smem + C::kQrOff);
    uint32_t* s_lut = reinterpret_cast<uint32_t*>(smem + C::kLutOff);
    float* s_red = reinterpret_cast<float*>(smem + C::kRedOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    const uint32_t b_full = smem_u32(bars), b_empty = b_full + 8 * S;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int G = p.group;
    const int64_t T = p.seq_lens ? static_cast<int64_t>(p.seq_lens[b]) : p.max_seq_len;
    const int64_t nchunks = (T + 15) / 16;
    const int64_t cps = (nchunks + p.num_splits - 1) / p.num_splits;
    const int64_t c_begin = split * cps;
    const int64_t c_end = (c_begin + cps < nchunks) ? c_begin + cps : nchunks;
    const int64_t ntiles = (c_end > c_begin) ? (c_end - c_begin + C::kWarps - 1) / C::kWarps : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(b_full + 8 * s, 1);
            mbar_init(b_empty + 8 * s, C::kWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < (1 << (2 * KB)); i += blockDim.x) s_lut[i] = p.pair_lut[i];
    __syncthreads();

    if (warp == C::kWarps) {
        // ------------------------------------------------------------------ bulk-copy producer
        if (lane == 0) {
            for (int64_t ti = 0; ti < ntiles; ++ti) {
                const int s = static_cast<int>(ti % S);
                if (!mbar_wait(b_empty + 8 * s, static_cast<uint32_t>((ti / S) & 1) ^ 1u, abort_flag)) break;
                const int64_t c0 = c_begin + ti * C::kWarps;
                const int nc = static_cast<int>((c_end - c0 < C::kWarps) ? c_end - c0 : C::kWarps);
                mbar_arrive_expect_tx(b_full + 8 * s, nc * C::kChunkBytes);
                uint8_t* st = smem + s * C::kStageBytes;
                for (int c = 0; c < nc; ++c) {
                    int64_t row0;
                    if (p.block_table)
                        row0 = (static_cast<int64_t>(p.block_table[static_cast<int64_t>(b) * p.max_blocks + c0 + c]) *
                                    p.num_kv_heads + h) * 16;
                    else
                        row0 = (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.max_seq_len + (c0 + c) * 16;
                    uint8_t* dst = st + c * C::kChunkBytes;
                    const uint32_t bar = b_full + 8 * s;
                    bulk_load(smem_u32(dst + C::kKOff), p.k_packed + row0 * C::kKRow, 16 * C::kKRow, bar);
                    bulk_load(smem_u32(dst + C::kNOff), p.k_norms + row0, 64, bar);
                    bulk_load(smem_u32(dst + C::kVOff), p.v_data + row0 * C::kVRow, 16 * C::kVRow, bar);
                    bulk_load(smem_u32(dst + C::kSOff), p.v_scales + row0 * G8, 32 * G8, bar);
                    bulk_load(smem_u32(dst + C::kZOff), p.v_zeros + row0 * G8, 32 * G8, bar);
                }
            }
            // drain: the last issued stages have landed before the CTA may reuse or leave them
            for (int64_t ti = (ntiles > S ? ntiles - S : 0); ti < ntiles; ++ti)
                mbar_wait_drain(b_full + 8 * static_cast<int>(ti % S), static_cast<uint32_t>((ti / S) & 1));
        }
    } else {
        // ------------------------------------------------------------------ rotate the query
        // q_rot[g][n] = sum_k q[g][k] Pi_op[n][k] on the tensor cores (fp16 inputs are exact products)
        const __half* qg = p.q + (static_cast<int64_t>(b) * p.num_q_heads + static_cast<int64_t>(h) * G) * D;
        for (int nt = warp; nt < NT; nt += C::kWarps) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int ks = 0; ks < KS; ++ks) {
                uint4 a = make_uint4(0u, 0u, 0u, 0u);
                if (gid < G) {
                    a.x = *reinterpret_cast<const uint32_t*>(qg + gid * D + 16 * ks + 2 * tig);
                    a.z = *reinterpret_cast<const uint32_t*>(qg + gid * D + 16 * ks + 2 * tig + 8);
                }
                const __half* prow = p.pi_op + (8 * nt + gid) * D + 16 * ks + 2 * tig;
                mma_f16(c, a, *reinterpret_cast<const uint32_t*>(prow), *reinterpret_cast<const uint32_t*>(prow + 8));
            }
            s_qr[gid * D + 8 * nt + 2 * tig] = c[0];
            s_qr[gid * D + 8 * nt + 2 * tig + 1] = c[1];
        }
        named_bar_sync(1, 32 * C::kWarps);
        // power-of-two prescale so the fp16 hi/lo halves of the scaled query stay in the normal range
        float amax = 0.f;
        for (int i = threadIdx.x; i < G * D; i += 32 * C::kWarps) amax = fmaxf(amax, fabsf(s_qr[i] * p.scale_log2));
#pragma unroll
        for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) s_red[warp] = amax;
        named_bar_sync(1, 32 * C::kWarps);
        amax = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
        int ex = 0;
        if (amax > 0.f) frexpf(amax, &ex);
        const float pre = (amax > 0.f) ? ldexpf(1.0f, 14 - ex) : 1.0f;     // max |q| * pre in [8192, 16384)
        const float unpre = 1.0f / pre;
        // score A fragments, coordinate-permuted so lane tig owns coords [tig*D/4, (tig+1)*D/4):
        // k-slots (2tig, 2tig+1, 2tig+8, 2tig+9) of k-step ks <- coords tig*D/4 + 4ks + (0, 1, 2, 3)
        for (int i = threadIdx.x; i < KS * 32; i += 32 * C::kWarps) {
            const int ks = i >> 5, ln = i & 31, g = ln >> 2, tg = ln & 3;
            const int c0 = tg * (D / 4) + 4 * ks;
            uint4 f = make_uint4(0u, 0u, 0u, 0u);
            if (g < G) {
                float x[4], hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[e] = s_qr[g * D + c0 + e] * p.scale_log2 * pre;
                    hi[e] = __half2float(__float2half_rn(x[e]));
                    lo[e] = x[e] - hi[e];
                }
                f.x = pack_f16(hi[0], hi[1]);
                f.y = pack_f16(lo[0], lo[1]);
                f.z = pack_f16(hi[2], hi[3]);
                f.w = pack_f16(lo[2], lo[3]);
            }
            s_qf[i] = f;
        }
        named_bar_sync(1, 32 * C::kWarps);

        // ------------------------------------------------------------------ token loop
        float o[NT][4];
#pragma unroll
        for (int m = 0; m < NT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
        float zacc[G8];
#pragma unroll
        for (int g = 0; g < G8; ++g) zacc[g] = 0.f;
        float m_run = -INFINITY, l_run = 0.f;

        for (int64_t ti = 0; ti < ntiles; ++ti) {
            const int s = static_cast<int>(ti % S);
            if (!mbar_wait(b_full + 8 * s, static_cast<uint32_t>((ti / S) & 1), abort_flag)) break;
            const int64_t chunk = c_begin + ti * C::kWarps + warp;
            if (chunk < c_end) {
                const uint8_t* ch = smem + s * C::kStageBytes + warp * C::kChunkBytes;
                // ---- scores: S'[16 x 8 tokens] per n-tile, rows gid (hi part) and gid+8 (lo part)
                float sc[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                    // this lane's quarter of the key row of token 8nt + gid
                    const uint8_t* krow = ch + C::kKOff + (8 * nt + gid) * C::kKRow;
                    uint32_t w[C::kQuarterWords];
                    if constexpr (C::kQuarterHalves % 2 == 0) {
                        const uint32_t* k32 = reinterpret_cast<const uint32_t*>(krow) + tig * (C::kQuarterHalves / 2);
#pragma unroll
                        for (int i = 0; i < C::kQuarterWords; ++i) w[i] = (2 * i < C::kQuarterHalves) ? k32[i] : 0u;
                    } else {
                        const uint16_t* k16 = reinterpret_cast<const uint16_t*>(krow) + tig * C::kQuarterHalves;
#pragma unroll
                        for (int i = 0; i < C::kQuarterWords; ++i) {
                            const uint32_t lo16 = (2 * i < C::kQuarterHalves) ? k16[2 * i] : 0u;
                            const uint32_t hi16 = (2 * i + 1 < C::kQuarterHalves) ? k16[2 * i + 1] : 0u;
                            w[i] = lo16 | (hi16 << 16);
                        }
                    }
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const uint4 a = s_qf[ks * 32 + lane];
                        const int bp = 4 * ks * KB;
                        uint32_t keys[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int bb = bp + 2 * e * KB;
                            const int wi = bb >> 5, sh = bb & 31;
                            uint32_t v = w[wi] >> sh;
                            if (sh + 2 * KB > 32) v |= w[wi + 1] << (32 - sh);
                            keys[e] = v & ((1u << (2 * KB)) - 1u);
                        }
                        mma_f16(sc[nt], a, s_lut[keys[0]], s_lut[keys[1]]);
                    }
                }
                // ---- logits (log2 domain) of head gid for tokens 2tig, 2tig+1, 8+2tig, 9+2tig
                const float* nrm = reinterpret_cast<const float*>(ch + C::kNOff);
                float lg[4];
                int tok[4] = {2 * tig, 2 * tig + 1, 8 + 2 * tig, 9 + 2 * tig};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int nt = e >> 1, k = e & 1;
                    const float raw = (sc[nt][k] + sc[nt][k + 2]) * unpre * nrm[tok[e]];
                    lg[e] = (chunk * 16 + tok[e] < T) ? raw : -INFINITY;
                }
                float mt = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
                const float m_new = fmaxf(m_run, mt);
                const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
                const float corr = exp2f(m_run - m_use);
                float pr[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) pr[e] = exp2f(lg[e] - m_use);
                l_run = l_run * corr + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
                m_run = m_new;
#pragma unroll
                for (int m = 0; m < NT; ++m) {
                    o[m][0] *= corr; o[m][1] *= corr; o[m][2] *= corr; o[m][3] *= corr;
                }
                // ---- values: per scale group, A = hi/lo of p * scale, B = integer codes
                const __half* vs = reinterpret_cast<const __half*>(ch + C::kSOff);
                const __half* vz = reinterpret_cast<const __half*>(ch + C::kZOff);
                const uint8_t* vrow[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) vrow[e] = ch + C::kVOff + tok[e] * C::kVRow;
#pragma unroll
                for (int g8 = 0; g8 < G8; ++g8) {
                    float wv[4];
                    float zs = 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        wv[e] = pr[e] * __half2float(vs[tok[e] * G8 + g8]);
                        zs = fmaf(pr[e], __half2float(vz[tok[e] * G8 + g8]), zs);
                    }
                    zacc[g8] = zacc[g8] * corr + zs;
                    uint4 a;
                    split_bf16(wv[0], wv[1], a.x, a.y);
                    split_bf16(wv[2], wv[3], a.z, a.w);
#pragma unroll
                    for (int mm = 0; mm < VG / 8; ++mm) {
                        const int m = g8 * (VG / 8) + mm;
                        const int col = 8 * m + gid;
                        const uint32_t b0 = vcode_pair<VB>(vrow[0], vrow[1], col);
                        const uint32_t b1 = vcode_pair<VB>(vrow[2], vrow[3], col);
                        mma_bf16(o[m], a, b0, b1);
                    }
                }
            } else {
                // no chunk for this warp in this stage: keep running statistics unchanged
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(b_empty + 8 * s);
        }

        // ------------------------------------------------------------------ per-warp finalisation
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
#pragma unroll
        for (int g8 = 0; g8 < G8; ++g8) {
            zacc[g8] += __shfl_xor_sync(0xffffffffu, zacc[g8], 1);
            zacc[g8] += __shfl_xor_sync(0xffffffffu, zacc[g8], 2);
        }
        // the stage ring is free once every consumer is past its last stage
        named_bar_sync(1, 32 * C::kWarps);
        float* comb = reinterpret_cast<float*>(smem);          // [warp][16 + 8D]
        float* mine = comb + warp * C::kPartFloats;
        if (tig == 0) {
            mine[gid] = m_run;
            mine[8 + gid] = l_run;
        }
#pragma unroll
        for (int m = 0; m < NT; ++m) {
            const int col = 8 * m + 2 * tig;
            const float z = zacc[(8 * m) / VG];
            mine[16 + gid * D + col] = o[m][0] + o[m][2] + z;
            mine[16 + gid * D + col + 1] = o[m][1] + o[m][3] + z;
        }
        named_bar_sync(1, 32 * C::kWarps);
        // ------------------------------------------------------------------ merge the four warps
        const int tid = threadIdx.x;
        float* part = p.partials +
                      ((static_cast<int64_t>(b) * p.num_kv_heads + h) * p.num_splits + split) * C::kPartFloats;
        for (int i = tid; i < G * D; i += 32 * C::kWarps) {
            const int g = i / D, col = i % D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, comb[w * C::kPartFloats + g]);
            const float Mu = (M == -INFINITY) ? 0.f : M;
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int w = 0; w < C::kWarps; ++w) {
                const float f = exp2f(comb[w * C::kPartFloats + g] - Mu);
                L += comb[w * C::kPartFloats + 8 + g] * f;
                O += comb[w * C::kPartFloats + 16 + g * D + col] * f;
            }
            if (p.num_splits == 1) {
                p.out[(static_cast<int64_t>(b) * p.num_q_heads + static_cast<int64_t>(h) * G + g) * D + col] =
                    (L > 0.f) ? O / L : 0.f;
            } else {
                part[16 + g * D + col] = O;
                if (col == 0) {
                    part[g] = M;
                    part[8 + g] = L;
                }
            }
        }
        if (p.num_splits > 1) {
            // ---------------------------------------------------------------- split-K merge, last CTA
            __threadfence();
            named_bar_sync(1, 32 * C::kWarps);
            int* ctr = p.counters + static_cast<int64_t>(b) * p.num_kv_heads + h;
            if (tid == 0) s_red[4] = __int_as_float(atomicAdd(ctr, 1));
            named_bar_sync(1, 32 * C::kWarps);
            if (__float_as_int(s_red[4]) == p.num_splits - 1) {
                __threadfence();
                const float* base =
                    p.partials + (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.num_splits * C::kPartFloats;
                for (int i = tid; i < G * D; i += 32 * C::kWarps) {
                    const int g = i / D, col = i % D;
                    float M = -INFINITY;
                    for (int sp = 0; sp < p.num_splits; ++sp) M = fmaxf(M, __ldcg(base + sp * C::kPartFloats + g));
                    const float Mu = (M == -INFINITY) ? 0.f : M;
                    float L = 0.f, O = 0.f;
                    for (int sp = 0; sp < p.num_splits; ++sp) {
                        const float* ps = base + sp * C::kPartFloats;
                        const float f = exp2f(__ldcg(ps + g) - Mu);
                        L += __ldcg(ps + 8 + g) * f;
                        O += __ldcg(ps + 16 + g * D + col) * f;
                    }
                    p.out[(static_cast<int64_t>(b) * p.num_q_heads + static_cast<int64_t>(h) * G + g) * D + col] =
                        (L > 0.f) ? O / L : 0.f;
                }
                if (tid == 0) *ctr = 0;      // leave the counter zeroed for the next call
            }
        }
    }
}

}  // namespace dev
}  // namespace tq
