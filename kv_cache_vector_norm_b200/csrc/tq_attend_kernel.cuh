// Fused decode-step attention over the compressed cache.
//
// "KV Cache API" (TurboQuant docs), store.py TurboQuantKVCache.attention_scores / attend: logits
// q . k * scale (scale 1/sqrt(head_dim) by default), softmax, weights @ dequantised values; the page
// materialises fp32 keys and values to do it.  "turbo-attn": the decode kernel is split-K over the paged
// cache and rotates the query once, so scores need no un-rotation.  Here neither keys nor values are
// ever materialised:
//   score_t = scale * n_t * <Pi_op q, c_op[idx_t]>       (tensor cores: fp16 codebook values x fp16
//                                                         hi/lo halves of the rotated query)
//   out     = sum_t p_t (q_t s_t + z_t) / sum_t p_t       (tensor cores: integer codes, exact as bf16
//                                                         subnormals, x bf16 hi/lo halves of p_t s_t;
//                                                         the zero term on FMAs)
// One CTA = one (split, kv head, sequence); warp 4 streams 16-token chunks of every pool array into a
// shared-memory ring with bulk TMA copies; warps 0..3 each consume one chunk of every stage with
// mma.sync fragments kept in registers; a second kernel merges the splits.
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
    uint4* qfrag;                                    // [B][H_kv][d/16 * 32 + 2]: score A fragments, 1 / prescale
    int num_splits;                                  // CTAs along the compressed sequence
    int num_parts;                                   // partials per (sequence, kv head): splits (+ 1 window)
    const __half* win_k;                             // nullable: [B][H_kv][win_max][d] recent keys, uncompressed
    const __half* win_v;
    const int32_t* win_lens;                         // nullable: win_max for every sequence
    int win_max;
    int qfrag_stride;                                // uint4 slots per (sequence, kv head) of qfrag
    // QJL residual keys (the kernels' QJL instantiations only)
    const uint8_t* k_signs;                          // pool of sign rows, d/8 bytes, LSB-first (1 = +1)
    const float* k_rho;                              // pool of residual norms
    const __half* s_op;                              // d x d sketch, row-major
    float s_scale_log2;                              // softmax scale * log2(e) * sqrt(pi/2) / d
    float s_row_bound;                               // max over rows of ||S_op row||
};

// Entries of the key table: a pair of codes -> half2 of codebook values up to 4 bits; from 5 bits (whose
// 2^(2 bits) pairs would not fit) one code -> its fp16 value in the low half, and a half2 takes two lookups.
template <int KB>
__host__ __device__ constexpr int key_table_entries() { return KB > 4 ? (1 << KB) : (1 << (2 * KB)); }

constexpr int kWinMax = 256;                         // largest window per (sequence, kv head)
constexpr int kWinChunk = 32;                        // window tokens staged in shared memory at a time

// shared memory of the window path (floats): query, scores, max/sum, one staged chunk, two partial sums
template <int D>
__host__ __device__ constexpr int window_smem_floats() {
    return 8 * D + 8 * kWinMax + 16 + kWinChunk * (D + 2) / 2 + 2 * 8 * D;
}

// uint4 slots per (sequence, kv head) of the query-fragment array: the fragments, then 1 / prescale of 8 heads
template <int D>
__host__ __device__ constexpr int qfrag_slots() { return (D / 16) * 32 + 2; }

template <int D, int KB, int VB, int VG, bool QJL = false>
struct AttCfg {
    static constexpr int kWarps = 4;                 // consumer warps
    static constexpr int kThreads = 32 * (kWarps + 1);
    static constexpr int kChunkTok = 16;             // tokens per chunk (= one paged block)
    static constexpr int kTileTok = kWarps * kChunkTok;
    // stages of the copy ring (a power of two): 4; 2 with the 32 KB table of 4-bit keys above d = 64, which keeps
    // four CTAs per SM resident (two 64-token stages of four CTAs still hold ~60 KB per SM in flight)
    static constexpr int kStages = (key_table_entries<KB>() * 128 > 8192 && D > 64) ? 2 : 4;
    // paged blocks of d = 64 are copied by the producer warp's lanes with cp.async, larger ones by bulk copies
    // from one lane (measured on the 64 x 4096-token paged cache: d = 64 99 vs 106 us, d = 128 162 vs 140 us)
    static constexpr bool kPagedCpAsync = (D == 64);
    static constexpr int kKRow = D * KB / 8;
    static constexpr int kVRow = D * VB / 8;
    static constexpr int kVGroups = D / VG;
    // one stage holds the tile's 64 tokens array by array; chunk c of an array starts at c * 16 rows
    static constexpr int kKOff = 0;
    static constexpr int kNOff = kKOff + kTileTok * kKRow;
    static constexpr int kVOff = kNOff + kTileTok * 4;
    static constexpr int kSOff = kVOff + kTileTok * kVRow;
    static constexpr int kZOff = kSOff + kTileTok * kVGroups * 2;
    // QJL: the sign rows (d/8 bytes) and residual norms of the tile follow the value arrays
    static constexpr int kSgRow = D / 8;
    static constexpr int kSgOff = kZOff + kTileTok * kVGroups * 2;
    static constexpr int kRhoOff = kSgOff + (QJL ? kTileTok * kSgRow : 0);
    static constexpr int kStageBytes = kRhoOff + (QJL ? kTileTok * 4 : 0);
    static constexpr int kQuarterBits = D * KB / 4;  // one lane's quarter of a key row (16-bit multiple)
    static constexpr int kQuarterHalves = kQuarterBits / 16;
    static constexpr int kQuarterWords = (kQuarterHalves + 1) / 2 + 1;
    static constexpr int kMinBlocks = (D == 256) ? 1 : 4;
    static constexpr int kPartFloats = 16 + 8 * D;
    // score A fragments from shared memory (one 16-byte load per k-step): keeping them in registers would
    // cost 32 registers and one resident CTA per SM
    static constexpr bool kQInRegs = false;
    // key table: a pair of codes (2 KB bits, first code in the low bits) -> half2 of codebook values, with one
    // copy per shared-memory bank (entry e of lane l at byte 128 e + 4 l), so lookups never conflict
    static constexpr int kPairs = key_table_entries<KB>();
    static constexpr int kLutBytes = kPairs * 128;
    // shared memory: stages | q fragments (d = 256) | key table (aligned to its size at run time) |
    // per-warp zero sums | barriers
    static constexpr int kCombineFloats = kWarps * kPartFloats;
    static constexpr int kRingBytes =
        (kStages * kStageBytes > kCombineFloats * 4) ? kStages * kStageBytes : kCombineFloats * 4;
    static constexpr int kQfOff = kRingBytes;
    static constexpr int kLutOff = kQfOff + (kQInRegs ? 0 : (QJL ? 2 : 1) * (D / 16) * 32 * 16);
    // tables up to 8 KB (key widths 1..3) start on a multiple of their size (slack reserved), so an entry's
    // address is (pair bits << 7) | lane bits; the 32 KB table of 4-bit keys would need 32 KB of slack and cost
    // resident CTAs, so it sits unaligned and its addresses are base + (pair bits << 7) + lane bits
    static constexpr bool kLutAligned = (kLutBytes <= 8192);
    // QJL: a table of the four sign pairs (two bits -> half2 of +-1), replicated per bank like the key table and
    // aligned to its 512 bytes (slack reserved)
    static constexpr int kSLutOff = kLutOff + (kLutAligned ? 2 : 1) * kLutBytes;
    static constexpr int kZsOff = kSLutOff + (QJL ? 1024 : 0);
    static constexpr int kBarOff = (kZsOff + kWarps * 8 * kVGroups * 4 + 15) & ~15;
    static constexpr int kSmemMain = kBarOff + 8 * (2 * kStages) + 16;
    // the window CTA reuses the same allocation
    static constexpr int kSmem = (kSmemMain > window_smem_floats<D>() * 4) ? kSmemMain : window_smem_floats<D>() * 4;
    static_assert(kNOff % 16 == 0 && kVOff % 16 == 0 && kSOff % 16 == 0 && kZOff % 16 == 0 && kSgOff % 16 == 0 &&
                      kRhoOff % 16 == 0 && kStageBytes % 16 == 0,
                  "bulk copies need 16-byte multiples");
    static_assert(VG % 32 == 0, "a 32-column slice of the value row lies in one scale group");
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

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// hi/lo bf16 split of two values: hi = x truncated to bf16 (the upper 16 bits), lo = bf16(x - hi);
// hi + lo is within 2^-16 |x| of x.  x - hi is exact; it is one packed f32x2 FMA (-1 * hi + x).
__device__ __forceinline__ void split_bf16(float2 x, uint32_t& hi, uint32_t& lo) {
    const uint32_t u0 = __float_as_uint(x.x), u1 = __float_as_uint(x.y);
    hi = __byte_perm(u0, u1, 0x7632);
    const float2 h = make_float2(__uint_as_float(u0 & 0xFFFF0000u), __uint_as_float(u1 & 0xFFFF0000u));
    const float2 r = __ffma2_rn(h, make_float2(-1.0f, -1.0f), x);
    lo = pack_bf16(r.x, r.y);
}

// n fp16 values at p (n in {1, 2, 4, 8}, naturally aligned) as floats
template <int N>
__device__ __forceinline__ void load_halves(const __half* p, float (&o)[N]) {
    if constexpr (N == 1) {
        o[0] = __half2float(p[0]);
    } else if constexpr (N == 2) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(p));
        o[0] = f.x; o[1] = f.y;
    } else if constexpr (N == 4) {
        const uint2 t = *reinterpret_cast<const uint2*>(p);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&t.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&t.y));
        o[0] = f0.x; o[1] = f0.y; o[2] = f1.x; o[3] = f1.y;
    } else {
        const uint4 t = *reinterpret_cast<const uint4*>(p);
        const uint32_t u[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
            o[2 * k] = f.x; o[2 * k + 1] = f.y;
        }
    }
}

// The little-endian bitstream `w` shifted right by `bit` (which may be as low as -31), low 32 bits.
template <int NW>
__device__ __forceinline__ uint32_t window_shr(const uint32_t (&w)[NW], int bit) {
    if (bit < 0) return w[0] << (-bit);
    const int wi = bit >> 5, sh = bit & 31;
    return sh ? __funnelshift_r(w[wi], w[wi + 1], sh) : w[wi];
}

// Value codes as bf16 operands without arithmetic.  A bf16 whose upper 8 bits are zero is exactly
// (its bits) * 2^-133 (subnormals, then the first normal binade with the same spacing), and the tensor cores
// take subnormal operands exactly; so masking the codes of two tokens out of `pr` (token a in bits 0..15,
// token b in 16..31) gives a register {code_a, code_b} * 2^(VB pos') * 2^-133, where the scale 2^(VB pos')
// depends only on the code's position and is divided out of the accumulator at the end.
// The lane field holds four codes, positions 0..3, VB bits apart (VB = 2, 3, 4).
template <int VB>
__device__ __forceinline__ uint32_t vcode_sel(uint32_t pr, int pos) {
    if constexpr (VB == 2) {
        return pr & (0x00030003u << (2 * pos));
    } else {
        constexpr uint32_t m = (1u << VB) - 1u, mm = m | (m << 16);
        return (pos < 2) ? (pr & (mm << (VB * pos))) : ((pr >> (2 * VB)) & (mm << (VB * (pos - 2))));
    }
}

// log2 of the position scale above: the accumulator row holding code position `pos` carries 2^(that)
template <int VB>
__host__ __device__ constexpr int vcode_scale_log2(int pos) {
    return (VB == 2) ? 2 * pos : ((VB == 8) ? 0 : VB * (pos & 1));
}

// The lane field of one token's value row for 32-column slice `sl`: the codes of columns
// 32 sl + 4 gid + (0..3), positions 0..3 (VB = 8: the four bytes).
template <int VB>
__device__ __forceinline__ uint32_t vfield(const uint8_t* row, int sl, int gid) {
    if constexpr (VB == 2) {
        return row[8 * sl + gid];
    } else if constexpr (VB == 4) {
        return *reinterpret_cast<const uint16_t*>(row + 16 * sl + 2 * gid);
    } else if constexpr (VB == 8) {
        return *reinterpret_cast<const uint32_t*>(row + 32 * sl + 4 * gid);
    } else {
        const int bit = 32 * VB * sl + 4 * VB * gid;
        const uint32_t* w = reinterpret_cast<const uint32_t*>(row) + (bit >> 5);
        return __funnelshift_r(w[0], w[1], bit & 31);
    }
}

// Tokens of sequence b that the compressed part attends to: seq_lens[b] (all max_seq_len tokens when seq_lens
// is NULL), clamped to [0, the tokens the layout can address] -- max_seq_len rows in the contiguous layout,
// max_blocks * 16 in the paged one -- so a length past the cache never reads past a sequence's rows or its
// block-table row.
__device__ __forceinline__ int64_t attend_seq_len(const AttendParams& p, int b) {
    const int64_t cap = p.block_table ? static_cast<int64_t>(p.max_blocks) * 16 : p.max_seq_len;
    const int64_t t = p.seq_lens ? static_cast<int64_t>(p.seq_lens[b]) : cap;
    return t < 0 ? 0 : (t > cap ? cap : t);
}

// The score B register of code positions j, j + 1 of the lane's key quarter w (j even): the table entry of the
// pair, or at 5..8 bits the two single entries merged (first code in the low half).  lane_addr: this lane's copy
// of the table; ALIGNED: the table starts on a multiple of its size, so an address is an OR of field and lane
// bits, else a sum.
template <int KB, bool ALIGNED, int NW>
__device__ __forceinline__ uint32_t key_b_reg(const uint32_t (&w)[NW], int j, uint32_t lane_addr) {
    if constexpr (KB > 4) {
        constexpr uint32_t kMask = ((1u << KB) - 1u) << 7;
        const uint32_t e0 = window_shr(w, j * KB - 7) & kMask, e1 = window_shr(w, (j + 1) * KB - 7) & kMask;
        const uint32_t v0 = ALIGNED ? lds_u32(lane_addr | e0) : lds_u32(lane_addr + e0);
        const uint32_t v1 = ALIGNED ? lds_u32(lane_addr | e1) : lds_u32(lane_addr + e1);
        return __byte_perm(v0, v1, 0x5410);
    } else {
        constexpr uint32_t kMask = ((1u << (2 * KB)) - 1u) << 7;
        const uint32_t e = window_shr(w, j * KB - 7) & kMask;
        return ALIGNED ? lds_u32(lane_addr | e) : lds_u32(lane_addr + e);
    }
}

// Query preparation: the rotated query q_rot[g] = Pi_op q[g] of each of the group's heads, scaled by softmax
// scale * log2(e) and a per-head power-of-two prescale, split into fp16 hi/lo halves and laid out as the score A
// fragments (rows gid = hi, gid + 8 = lo); slots d/16 * 32 and + 1 hold 1 / prescale of heads 0..7.
// The prescale comes from a bound, |q_rot_j| <= ||Pi_op|| ||q|| < 1.0625 ||q||, so max |x * pre| < 2^15 and
// no reduction over q_rot is needed: CTA x of grid (d / 32, H_kv, B) computes n-tiles 4x .. 4x + 3 (one per
// warp) and writes their fragments straight from the MMA accumulators.  The attention grid is its
// programmatic dependent.
// With QJL residual keys the grid is (2 d / 32, H_kv, B): CTAs x >= d / 32 prepare, the same way, the sketched
// query S_op q scaled by softmax scale * log2(e) * sqrt(pi/2) / d (the estimator's factor), whose bound is
// ||S_op row||_max ||q||, into a second block of fragments.
constexpr int kPrepThreads = 128;

template <int D>
__global__ void __launch_bounds__(kPrepThreads) attend_prep_kernel(const AttendParams p) {
    constexpr int KS = D / 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const bool sketch = blockIdx.x >= D / 32;                   // the QJL block: S_op q
    const int bx = sketch ? blockIdx.x - D / 32 : blockIdx.x;
    const int nt = bx * (kPrepThreads / 32) + warp;             // n-tile: columns 8 nt .. 8 nt + 7
    const int h = blockIdx.y, b = blockIdx.z;
    const int G = p.group;
    uint4* qf = p.qfrag + (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.qfrag_stride +
                (sketch ? qfrag_slots<D>() : 0);
    const __half* mat = sketch ? p.s_op : p.pi_op;
    const float scale_log2 = sketch ? p.s_scale_log2 : p.scale_log2;
    const float mat_bound = sketch ? p.s_row_bound : 1.0625f;
    // the attention grid may be scheduled at once and start streaming the cache; its consumers wait for this
    // grid's completion (griddepcontrol.wait) before they read the fragments
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const __half* qg = p.q + (static_cast<int64_t>(b) * p.num_q_heads + static_cast<int64_t>(h) * G) * D;
    // every fragment is loaded before the first MMA, so the loads overlap
    uint32_t bf[KS][2], af[KS][2];
    const __half* prow = mat + (8 * nt + gid) * D + 2 * tig;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        bf[ks][0] = __ldg(reinterpret_cast<const uint32_t*>(prow + 16 * ks));
        bf[ks][1] = __ldg(reinterpret_cast<const uint32_t*>(prow + 16 * ks + 8));
        af[ks][0] = (gid < G) ? __ldg(reinterpret_cast<const uint32_t*>(qg + gid * D + 16 * ks + 2 * tig)) : 0u;
        af[ks][1] = (gid < G) ? __ldg(reinterpret_cast<const uint32_t*>(qg + gid * D + 16 * ks + 2 * tig + 8)) : 0u;
    }
    // ||q_gid||^2 from the fragments this quad holds (lane tig: coordinates 16 ks + 2 tig + {0, 1, 8, 9})
    float ss = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&af[ks][j]));
            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
        }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const float bound = sqrtf(ss) * fabsf(scale_log2) * mat_bound;
    // bound = m 2^ex with m in [0.5, 1); pre = 2^(14 - ex), so |x| * pre < 2^15 (zero or tiny queries clamped)
    int ex = static_cast<int>((__float_as_uint(bound) >> 23) & 255u) - 126;
    ex = (bound > 0.f) ? max(ex, -100) : 14;
    const float pre = __uint_as_float(static_cast<uint32_t>(127 + 14 - ex) << 23);
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) mma_f16(c, make_uint4(af[ks][0], 0u, af[ks][1], 0u), bf[ks][0], bf[ks][1]);
    // c0, c1 = q_rot[gid][8 nt + 2 tig + {0, 1}]; the fragment of (head gid, k-step ks) holds coordinates
    // tg * D/4 + 4 ks + (0..3), so columns 8 nt .. + 3 and + 4 .. + 7 are two whole fragments: lanes tig = 0, 2
    // assemble them with the halves of lanes tig = 1, 3
    float hi[2], lo[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const float x = c[e] * scale_log2 * pre;
        hi[e] = __half2float(__float2half_rn(x));
        lo[e] = x - hi[e];
    }
    const uint32_t h01 = pack_f16(hi[0], hi[1]), l01 = pack_f16(lo[0], lo[1]);
    const uint32_t h23 = __shfl_down_sync(0xffffffffu, h01, 1), l23 = __shfl_down_sync(0xffffffffu, l01, 1);
    if ((tig & 1) == 0) {
        const int col = 8 * nt + 2 * tig;                         // first of this fragment's four coordinates
        const int tg = col / (D / 4), ks = (col % (D / 4)) / 4;
        qf[ks * 32 + gid * 4 + tg] = make_uint4(h01, l01, h23, l23);
    }
    if (bx == 0 && warp == 0 && tig == 0) reinterpret_cast<float*>(qf + KS * 32)[gid] = 1.0f / pre;
}

// The window part of one (sequence, kv head): scores of the group's queries against the recent uncompressed
// keys (fp32 dot products of the fp16 inputs, in the log2 domain like the compressed part's), their maximum m,
// l = sum 2^(s - m) and O = sum 2^(s - m) v -- one partial of the split merge.  All threads of the CTA.  Keys
// and values go through shared memory in chunks of kWinChunk tokens, loaded with coalesced 16-byte reads; key
// rows are padded by 4 bytes so the per-token dot products read distinct banks.
template <int D>
__device__ void attend_window_partial(const AttendParams& p, int b, int h, uint8_t* smem, float* part) {
    const int G = p.group, tid = threadIdx.x, nth = blockDim.x, warp = tid >> 5, lane = tid & 31;
    constexpr int KR = D + 2;                              // padded key row, in halves
    float* qs = reinterpret_cast<float*>(smem);            // [8][D]  query * scale * log2(e)
    float* ss = qs + 8 * D;                                // [8][kWinMax]  scores, then weights
    float* ml = ss + 8 * kWinMax;                          // [16]  per-head max and sum
    __half* kv = reinterpret_cast<__half*>(ml + 16);       // one chunk of keys [kWinChunk][KR] or values [kWinChunk][D]
    float* red = ml + 16 + kWinChunk * KR / 2;             // [2][8][D] partial sums of up to two token groups
    int L = p.win_lens ? p.win_lens[b] : p.win_max;
    L = L < 0 ? 0 : (L > p.win_max ? p.win_max : L);
    const __half* qg = p.q + (static_cast<int64_t>(b) * p.num_q_heads + static_cast<int64_t>(h) * G) * D;
    const int64_t base = (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.win_max * D;
    const __half* wk = p.win_k + base;
    const __half* wv = p.win_v + base;
    for (int i = tid; i < G * D; i += nth) qs[i] = __half2float(qg[i]) * p.scale_log2;
    // ---- scores, chunk by chunk: thread (g, t) of the chunk
    for (int t0 = 0; t0 < L; t0 += kWinChunk) {
        const int cl = (L - t0 < kWinChunk) ? L - t0 : kWinChunk;
        __syncthreads();                                   // the previous chunk's readers are done (and qs is set)
        for (int i = tid; i < cl * (D / 8); i += nth) {
            const int t = i / (D / 8), c8 = i % (D / 8);
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(wk + static_cast<int64_t>(t0 + t) * D) + c8);
            uint32_t* dst = reinterpret_cast<uint32_t*>(kv + t * KR + 8 * c8);
            dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
        }
        __syncthreads();
        for (int i = tid; i < G * cl; i += nth) {
            const int g = i / cl, t = i % cl;
            const __half2* kr = reinterpret_cast<const __half2*>(kv + t * KR);
            const float2* qr = reinterpret_cast<const float2*>(qs + g * D);
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
            for (int c = 0; c < D / 2; ++c) {
                const float2 k2 = __half22float2(kr[c]);
                const float2 q2 = qr[c];
                acc0 = fmaf(q2.x, k2.x, acc0);
                acc1 = fmaf(q2.y, k2.y, acc1);
            }
            ss[g * kWinMax + t0 + t] = acc0 + acc1;
        }
    }
    __syncthreads();
    // ---- per head: max, weights 2^(s - m), their sum
    for (int g = warp; g < G; g += nth / 32) {
        float m = -INFINITY;
        for (int t = lane; t < L; t += 32) m = fmaxf(m, ss[g * kWinMax + t]);
#pragma unroll
        for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
        for (int t = lane; t < L; t += 32) {
            const float w = exp2f(ss[g * kWinMax + t] - m);
            ss[g * kWinMax + t] = w;
            l += w;
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            ml[g] = m;
            ml[8 + g] = l;
        }
    }
    // ---- O = sum_t w_t v_t: thread (grp, c2) accumulates column pair c2 of every head over every ngrp-th token
    const int ngrp = (nth / (D / 2) >= 2) ? 2 : 1;
    const int grp = tid / (D / 2), c2 = tid % (D / 2);
    float acc[8][2];
#pragma unroll
    for (int g = 0; g < 8; ++g) acc[g][0] = acc[g][1] = 0.f;
    for (int t0 = 0; t0 < L; t0 += kWinChunk) {
        const int cl = (L - t0 < kWinChunk) ? L - t0 : kWinChunk;
        __syncthreads();
        for (int i = tid; i < cl * (D / 8); i += nth) {
            const int t = i / (D / 8), c8 = i % (D / 8);
            reinterpret_cast<uint4*>(kv + t * D)[c8] =
                __ldg(reinterpret_cast<const uint4*>(wv + static_cast<int64_t>(t0 + t) * D) + c8);
        }
        __syncthreads();
        if (grp < ngrp) {
            for (int t = grp; t < cl; t += ngrp) {
                const float2 v2 = __half22float2(reinterpret_cast<const __half2*>(kv + t * D)[c2]);
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    if (g < G) {
                        const float w = ss[g * kWinMax + t0 + t];
                        acc[g][0] = fmaf(w, v2.x, acc[g][0]);
                        acc[g][1] = fmaf(w, v2.y, acc[g][1]);
                    }
                }
            }
        }
    }
    if (grp < ngrp) {
#pragma unroll
        for (int g = 0; g < 8; ++g) reinterpret_cast<float2*>(red + (grp * 8 + g) * D)[c2] = make_float2(acc[g][0], acc[g][1]);
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += nth) {
        const int g = i / D, c = i % D;
        part[16 + g * D + c] = (ngrp == 2) ? red[g * D + c] + red[(8 + g) * D + c] : red[g * D + c];
    }
    if (tid < G) {
        part[tid] = ml[tid];
        part[8 + tid] = ml[8 + tid];
    }
}

// Fused decode attention for one (split, kv head, sequence).  Per 16-token chunk and warp:
//   scores  S[head][tok]  = (q hi/lo, fp16 A, rows gid / gid + 8) x (codebook pairs, fp16 B) on mma.sync
//   values  O^T[col][head] += (value codes, bf16 A, exact) x (hi/lo of p * scale, bf16 B)
// so each lane's probabilities (head gid, tokens 2tig, 2tig+1, 2tig+8, 2tig+9) are already the B fragment
// of the value product, and the accumulator is D/16 x 4 registers.
// QJL: the keys are QJL residual keys; each chunk adds a second score contraction, the sketched query S_op q
// against the keys' sign bits as +-1 pairs, weighted by the key's residual norm.
template <int D, int KB, int VB, int VG, bool QJL = false>
__global__ void __launch_bounds__(AttCfg<D, KB, VB, VG, QJL>::kThreads, AttCfg<D, KB, VB, VG, QJL>::kMinBlocks)
    attend_kernel(const AttendParams p) {
    using C = AttCfg<D, KB, VB, VG, QJL>;
    constexpr int S = C::kStages;
    constexpr int KS = D / 16;                        // k-steps of the score contraction
    constexpr int MT = D / 16;                        // m-tiles (16 value columns) of the value contraction
    constexpr int NSL = D / 32;                       // 32-column slices (two m-tiles)
    constexpr int G8 = C::kVGroups;
    // probabilities enter the value product as p * 2^kPExp so that p * scale * code * 2^-133 stays normal
    constexpr int kPExp = 80;
    extern __shared__ __align__(16) uint8_t smem[];
    uint4* s_qf = reinterpret_cast<uint4*>(smem + C::kQfOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    const uint32_t b_full = smem_u32(bars), b_empty = b_full + 8 * S;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S);
    // small key tables start on a multiple of their size, so an entry's address is (entry << 7) | lane bits
    const uint32_t lut_addr = C::kLutAligned
        ? (smem_u32(smem + C::kLutOff) + C::kLutBytes - 1) & ~static_cast<uint32_t>(C::kLutBytes - 1)
        : smem_u32(smem + C::kLutOff);
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + (lut_addr - smem_u32(smem)));
    const uint32_t slut_addr = (smem_u32(smem + C::kSLutOff) + 511u) & ~511u;    // QJL sign pairs

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int G = p.group;
    static_assert(window_smem_floats<D>() * 4 <= C::kSmem, "the window path fits the CTA's shared memory");
    static_assert(C::kThreads >= D / 2, "one thread per column pair in the window's value pass");
    if (split == p.num_splits) {
        // the extra CTA of a call with a window of recent uncompressed tokens: its own partial, then done
        attend_window_partial<D>(p, b, h, smem,
                                 p.partials + ((static_cast<int64_t>(b) * p.num_kv_heads + h) * p.num_parts + split) *
                                                  C::kPartFloats);
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        return;
    }
    const int64_t T = attend_seq_len(p, b);
    const int64_t nchunks = (T + 15) / 16;
    const int64_t cps = (nchunks + p.num_splits - 1) / p.num_splits;
    const int64_t c_begin = split * cps;
    const int64_t c_end = (c_begin + cps < nchunks) ? c_begin + cps : nchunks;
    const int64_t ntiles = (c_end > c_begin) ? (c_end - c_begin + C::kWarps - 1) / C::kWarps : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // one expect-tx arrival by lane 0, or one cp.async arrival per lane of the producer warp (paged)
            mbar_init(b_full + 8 * s, (p.block_table && C::kPagedCpAsync) ? 32 : 1);
            mbar_init(b_empty + 8 * s, C::kWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    // the producer issues its first copies as soon as the barriers exist; the consumers fill the code-pair table
    // (its global load overlaps those copies) and publish it with their own named barrier
    __syncthreads();

    if (warp == C::kWarps) {
        // ------------------------------------------------------------------ copy producer
        if (!p.block_table) {
            // contiguous cache: a stage's chunks are consecutive rows of the pool, one bulk copy per array (lane 0)
            if (lane == 0) {
                for (int64_t ti = 0; ti < ntiles; ++ti) {
                    const int s = static_cast<int>(ti % S);
                    if (!mbar_wait(b_empty + 8 * s, static_cast<uint32_t>((ti / S) & 1) ^ 1u, abort_flag)) break;
                    const int64_t c0 = c_begin + ti * C::kWarps;
                    const int nc = static_cast<int>((c_end - c0 < C::kWarps) ? c_end - c0 : C::kWarps);
                    uint8_t* st = smem + s * C::kStageBytes;
                    const uint32_t bar = b_full + 8 * s;
                    mbar_arrive_expect_tx(bar, nc * (C::kStageBytes / C::kWarps));
                    const int64_t row0 = (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.max_seq_len + c0 * 16;
                    const int rows = nc * 16;
                    bulk_load(smem_u32(st + C::kKOff), p.k_packed + row0 * C::kKRow, rows * C::kKRow, bar);
                    bulk_load(smem_u32(st + C::kNOff), p.k_norms + row0, rows * 4, bar);
                    bulk_load(smem_u32(st + C::kVOff), p.v_data + row0 * C::kVRow, rows * C::kVRow, bar);
                    bulk_load(smem_u32(st + C::kSOff), p.v_scales + row0 * G8, rows * G8 * 2, bar);
                    bulk_load(smem_u32(st + C::kZOff), p.v_zeros + row0 * G8, rows * G8 * 2, bar);
                    if constexpr (QJL) {
                        bulk_load(smem_u32(st + C::kSgOff), p.k_signs + row0 * C::kSgRow, rows * C::kSgRow, bar);
                        bulk_load(smem_u32(st + C::kRhoOff), p.k_rho + row0, rows * 4, bar);
                    }
                }
                for (int64_t ti = (ntiles > S ? ntiles - S : 0); ti < ntiles; ++ti)
                    mbar_wait_drain(b_full + 8 * static_cast<int>(ti % S), static_cast<uint32_t>((ti / S) & 1));
            }
        } else if constexpr (C::kPagedCpAsync) {
            // paged cache, d = 64: every 16-token block is a separate small piece of each array, and a run of
            // small bulk copies from one thread is serial, so the whole warp copies a stage in 16-byte cp.async
            // pieces and each lane arrives on the stage's barrier once its pieces have landed.  The block indices
            // of 32 chunks are read at once (one per lane), a period ahead of their use.
            static_assert(32 % C::kWarps == 0, "a stage's chunks lie in one 32-chunk period of block indices");
            const int32_t* bt = p.block_table + static_cast<int64_t>(b) * p.max_blocks;
            auto block_at = [&](int64_t rel) -> int32_t {      // block index of the split's chunk rel (0 past the end)
                return (c_begin + rel < c_end) ? __ldg(bt + c_begin + rel) : 0;
            };
            int32_t blk_cur = block_at(lane), blk_next = block_at(32 + lane);
            for (int64_t ti = 0; ti < ntiles; ++ti) {
                const int s = static_cast<int>(ti % S);
                const int64_t rel0 = ti * C::kWarps;            // the stage's first chunk, split-relative
                if (ti > 0 && (rel0 & 31) == 0) {
                    blk_cur = blk_next;
                    blk_next = block_at(rel0 + 32 + lane);
                }
                const bool ok =
                    (lane != 0) || mbar_wait(b_empty + 8 * s, static_cast<uint32_t>((ti / S) & 1) ^ 1u, abort_flag);
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
                const int64_t c0 = c_begin + rel0;
                const int nc = static_cast<int>((c_end - c0 < C::kWarps) ? c_end - c0 : C::kWarps);
                const uint32_t st_addr = smem_u32(smem + s * C::kStageBytes);
                int32_t blks[C::kWarps];
#pragma unroll
                for (int c = 0; c < C::kWarps; ++c)
                    blks[c] = __shfl_sync(0xffffffffu, blk_cur, static_cast<int>(rel0 & 31) + c);
                auto blk_of = [&](int c) -> int32_t {
                    int32_t v = blks[0];
#pragma unroll
                    for (int k = 1; k < C::kWarps; ++k) v = (c == k) ? blks[k] : v;
                    return v;
                };
                // an array of R-byte rows holds a block as 16 R contiguous bytes: R pieces of 16 bytes
                auto copy_array = [&](uint32_t off, const void* base, int R) {
                    for (int i = lane; i < nc * R; i += 32) {
                        const int c = i / R, piece = i - c * R;
                        const int64_t row0 = (static_cast<int64_t>(blk_of(c)) * p.num_kv_heads + h) * 16;
                        cp_async16(st_addr + off + static_cast<uint32_t>(c * 16 * R + piece * 16),
                                   static_cast<const uint8_t*>(base) + row0 * R + piece * 16);
                    }
                };
                copy_array(C::kKOff, p.k_packed, C::kKRow);
                copy_array(C::kNOff, p.k_norms, 4);
                copy_array(C::kVOff, p.v_data, C::kVRow);
                copy_array(C::kSOff, p.v_scales, 2 * G8);
                copy_array(C::kZOff, p.v_zeros, 2 * G8);
                if constexpr (QJL) {
                    copy_array(C::kSgOff, p.k_signs, C::kSgRow);
                    copy_array(C::kRhoOff, p.k_rho, 4);
                }
                cp_async_arrive_noinc(b_full + 8 * s);
            }
            if (lane == 0)
                for (int64_t ti = (ntiles > S ? ntiles - S : 0); ti < ntiles; ++ti)
                    mbar_wait_drain(b_full + 8 * static_cast<int>(ti % S), static_cast<uint32_t>((ti / S) & 1));
        } else if (lane == 0) {
            // paged cache, larger blocks: one bulk copy per array and block, from lane 0
            for (int64_t ti = 0; ti < ntiles; ++ti) {
                const int s = static_cast<int>(ti % S);
                if (!mbar_wait(b_empty + 8 * s, static_cast<uint32_t>((ti / S) & 1) ^ 1u, abort_flag)) break;
                const int64_t c0 = c_begin + ti * C::kWarps;
                const int nc = static_cast<int>((c_end - c0 < C::kWarps) ? c_end - c0 : C::kWarps);
                uint8_t* st = smem + s * C::kStageBytes;
                const uint32_t bar = b_full + 8 * s;
                mbar_arrive_expect_tx(bar, nc * (C::kStageBytes / C::kWarps));
                for (int c = 0; c < nc; ++c) {
                    const int64_t blk = p.block_table[static_cast<int64_t>(b) * p.max_blocks + c0 + c];
                    const int64_t row0 = (blk * p.num_kv_heads + h) * 16;
                    bulk_load(smem_u32(st + C::kKOff + c * 16 * C::kKRow), p.k_packed + row0 * C::kKRow,
                              16 * C::kKRow, bar);
                    bulk_load(smem_u32(st + C::kNOff + c * 64), p.k_norms + row0, 64, bar);
                    bulk_load(smem_u32(st + C::kVOff + c * 16 * C::kVRow), p.v_data + row0 * C::kVRow,
                              16 * C::kVRow, bar);
                    bulk_load(smem_u32(st + C::kSOff + c * 32 * G8), p.v_scales + row0 * G8, 32 * G8, bar);
                    bulk_load(smem_u32(st + C::kZOff + c * 32 * G8), p.v_zeros + row0 * G8, 32 * G8, bar);
                    if constexpr (QJL) {
                        bulk_load(smem_u32(st + C::kSgOff + c * 16 * C::kSgRow), p.k_signs + row0 * C::kSgRow,
                                  16 * C::kSgRow, bar);
                        bulk_load(smem_u32(st + C::kRhoOff + c * 64), p.k_rho + row0, 64, bar);
                    }
                }
            }
            for (int64_t ti = (ntiles > S ? ntiles - S : 0); ti < ntiles; ++ti)
                mbar_wait_drain(b_full + 8 * static_cast<int>(ti % S), static_cast<uint32_t>((ti / S) & 1));
        }
    } else {
        // ------------------------------------------------------------------ query fragments
        // written by attend_prep_kernel, the grid this one depends on programmatically
        fill_replicated_by(lut, p.pair_lut, C::kPairs, threadIdx.x, 32 * C::kWarps);
        if constexpr (QJL) {
            // entry e = two sign bits (first coordinate in bit 0) -> half2 of +-1 (1 = +1), per bank as above
            if (threadIdx.x < 4 * 32) {
                const uint32_t e = threadIdx.x >> 5;
                const uint32_t v = ((e & 1u) ? 0x3C00u : 0xBC00u) | (((e & 2u) ? 0x3C00u : 0xBC00u) << 16);
                reinterpret_cast<uint32_t*>(smem + (slut_addr - smem_u32(smem)))[threadIdx.x] = v;
            }
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint4* qf = p.qfrag + (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.qfrag_stride;
        const float unpre = __ldcg(reinterpret_cast<const float*>(qf + KS * 32) + gid);   // head gid's
        float unpre2 = 0.f;
        if constexpr (QJL) unpre2 = __ldcg(reinterpret_cast<const float*>(qf + qfrag_slots<D>() + KS * 32) + gid);
        if constexpr (!C::kQInRegs) {
            for (int i = threadIdx.x; i < KS * 32; i += 32 * C::kWarps) s_qf[i] = __ldcg(qf + i);
            if constexpr (QJL)
                for (int i = threadIdx.x; i < KS * 32; i += 32 * C::kWarps)
                    s_qf[KS * 32 + i] = __ldcg(qf + qfrag_slots<D>() + i);
        }
        named_bar_sync(1, 32 * C::kWarps);              // the table and the query fragments are in place

        // ------------------------------------------------------------------ token loop
        uint4 qa[C::kQInRegs ? KS : 1];
        if constexpr (C::kQInRegs) {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) qa[ks] = __ldcg(qf + ks * 32 + lane);
        }
        const uint32_t lane_addr = lut_addr + 4u * lane;
        float o[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
        float zacc[G8];
#pragma unroll
        for (int g = 0; g < G8; ++g) zacc[g] = 0.f;
        // Lazy running maximum: the probabilities are 2^(logit - m_off) with m_off = m_run - kPExp, and m_run moves
        // only when a logit exceeds m_run + kSlack (then every accumulator is rescaled once); in between, p may
        // reach 2^(kSlack + kPExp), which fp32 and the bf16 operands hold with ample room.
        constexpr float kSlack = 8.f;
        float m_run = -INFINITY, m_thr = -INFINITY, m_off = 0.f, l_run = 0.f;
        // this lane's byte offsets inside one stage: its quarter of key rows gid and 8 + gid, its tokens' norms,
        // scale / zero rows and value fields
        const uint8_t* const st0 = smem + warp * 16 * C::kKRow + gid * C::kKRow + tig * (C::kQuarterBits / 8);
        const int t0 = 2 * tig;                        // tokens t0, t0 + 1, t0 + 8, t0 + 9 of the chunk
        const int o_nrm = C::kNOff + (warp * 16 + t0) * 4;
        const int o_scl = C::kSOff + (warp * 16 + t0) * G8 * 2;
        const int o_zer = C::kZOff + (warp * 16 + t0) * G8 * 2;
        const int o_val = C::kVOff + (warp * 16 + t0) * C::kVRow;

        // 32-bit loop state: a split holds fewer than 2^31 chunks
        const int ntiles32 = static_cast<int>(ntiles);
        const int nrel = static_cast<int>(c_end - c_begin);
        // tokens of the split's last chunk that belong to the sequence (16 for every other chunk)
        const int last_valid = static_cast<int>(T - (c_end - 1) * 16);
        for (int ti = 0; ti < ntiles32; ++ti) {
            const int s = ti & (S - 1);
            if (!mbar_wait(b_full + 8 * s, static_cast<uint32_t>((ti / S) & 1), abort_flag)) break;
            const int rel = ti * C::kWarps + warp;        // chunk index within the split
            if (rel < nrel) {
                const uint8_t* const stg = smem + s * C::kStageBytes;
                const uint8_t* const kch = st0 + s * C::kStageBytes;
                // ---- scores: S'[16 x 8 tokens] per n-tile, rows gid (hi part) and gid+8 (lo part)
                uint32_t w[2][C::kQuarterWords];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const uint8_t* krow = kch + 8 * nt * C::kKRow;
                    if constexpr (C::kQuarterHalves % 2 == 0) {
                        const uint32_t* k32 = reinterpret_cast<const uint32_t*>(krow);
#pragma unroll
                        for (int i = 0; i < C::kQuarterWords; ++i) w[nt][i] = (2 * i < C::kQuarterHalves) ? k32[i] : 0u;
                    } else {
                        const uint16_t* k16 = reinterpret_cast<const uint16_t*>(krow);
#pragma unroll
                        for (int i = 0; i < C::kQuarterWords; ++i) {
                            const uint32_t lo16 = (2 * i < C::kQuarterHalves) ? k16[2 * i] : 0u;
                            const uint32_t hi16 = (2 * i + 1 < C::kQuarterHalves) ? k16[2 * i + 1] : 0u;
                            w[nt][i] = lo16 | (hi16 << 16);
                        }
                    }
                }
                float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    uint4 a;
                    if constexpr (C::kQInRegs) a = qa[ks]; else a = s_qf[ks * 32 + lane];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        // code pairs (4ks, 4ks+1) and (4ks+2, 4ks+3) of the lane's quarter
                        mma_f16(sc[nt], a, key_b_reg<KB, C::kLutAligned>(w[nt], 4 * ks, lane_addr),
                                key_b_reg<KB, C::kLutAligned>(w[nt], 4 * ks + 2, lane_addr));
                    }
                }
                // ---- logits (log2 domain) of head gid for tokens t0, t0+1, t0+8, t0+9
                const float2 n01 = *reinterpret_cast<const float2*>(stg + o_nrm);
                const float2 n89 = *reinterpret_cast<const float2*>(stg + o_nrm + 32);
                float lg[4];
                {
                    const float2 u2 = make_float2(unpre, unpre);
                    const float2 r0 = __fmul2_rn(__fadd2_rn(make_float2(sc[0][0], sc[0][1]), make_float2(sc[0][2], sc[0][3])),
                                                 __fmul2_rn(n01, u2));
                    const float2 r1 = __fmul2_rn(__fadd2_rn(make_float2(sc[1][0], sc[1][1]), make_float2(sc[1][2], sc[1][3])),
                                                 __fmul2_rn(n89, u2));
                    lg[0] = r0.x; lg[1] = r0.y; lg[2] = r1.x; lg[3] = r1.y;
                }
                if constexpr (QJL) {
                    // QJL term: rho_t * <S_op q, signs_t> (the prepared fragments carry scale log2(e) sqrt(pi/2)/d);
                    // this lane's quarter of the sign row of token 8 nt + gid holds coordinates tig d/4 ..
                    constexpr int kSW = (D / 4 + 31) / 32;
                    uint32_t sw[2][kSW + 1];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const uint8_t* srow = stg + C::kSgOff + (warp * 16 + 8 * nt + gid) * C::kSgRow + tig * (D / 32);
                        if constexpr (D == 64) {
                            sw[nt][0] = *reinterpret_cast<const uint16_t*>(srow);
                        } else {
#pragma unroll
                            for (int i = 0; i < kSW; ++i) sw[nt][i] = reinterpret_cast<const uint32_t*>(srow)[i];
                        }
                        sw[nt][kSW] = 0u;
                    }
                    const uint32_t slane = slut_addr + 4u * lane;
                    float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const uint4 a = s_qf[KS * 32 + ks * 32 + lane];
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            const uint32_t e0 = window_shr(sw[nt], 4 * ks - 7) & (3u << 7);
                            const uint32_t e1 = window_shr(sw[nt], 4 * ks + 2 - 7) & (3u << 7);
                            mma_f16(s2[nt], a, lds_u32(slane | e0), lds_u32(slane | e1));
                        }
                    }
                    const float2 rh01 = *reinterpret_cast<const float2*>(stg + C::kRhoOff + (warp * 16 + t0) * 4);
                    const float2 rh89 = *reinterpret_cast<const float2*>(stg + C::kRhoOff + (warp * 16 + t0 + 8) * 4);
                    lg[0] = fmaf((s2[0][0] + s2[0][2]) * unpre2, rh01.x, lg[0]);
                    lg[1] = fmaf((s2[0][1] + s2[0][3]) * unpre2, rh01.y, lg[1]);
                    lg[2] = fmaf((s2[1][0] + s2[1][2]) * unpre2, rh89.x, lg[2]);
                    lg[3] = fmaf((s2[1][1] + s2[1][3]) * unpre2, rh89.y, lg[3]);
                }
                if (rel == nrel - 1 && last_valid < 16) {          // the sequence's last, partial chunk
                    lg[0] = (t0 < last_valid) ? lg[0] : -INFINITY;
                    lg[1] = (t0 + 1 < last_valid) ? lg[1] : -INFINITY;
                    lg[2] = (t0 + 8 < last_valid) ? lg[2] : -INFINITY;
                    lg[3] = (t0 + 9 < last_valid) ? lg[3] : -INFINITY;
                }
                const float lm = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
                if (__any_sync(0xffffffffu, lm > m_thr)) {
                    // a logit passed its head's threshold: move that head's maximum and rescale everything once
                    float mq = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, 1));
                    mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, 2));
                    if (mq > m_thr) {
                        const float corr = ex2(m_run - mq);                  // 0 while m_run is -inf
                        m_run = mq;
                        m_thr = mq + kSlack;
                        m_off = mq - static_cast<float>(kPExp);
                        l_run *= corr;
#pragma unroll
                        for (int g = 0; g < G8; ++g) zacc[g] *= corr;
                        // stash the factor for the lanes holding this head's accumulator columns
                        mq = corr;
                    } else {
                        mq = 1.f;
                    }
                    // the accumulator columns are heads 2tig and 2tig+1: their factors sit in lanes 8tig, 8tig+4
                    const float ca = __shfl_sync(0xffffffffu, mq, 8 * tig);
                    const float cb = __shfl_sync(0xffffffffu, mq, 8 * tig + 4);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        o[m][0] *= ca; o[m][1] *= cb; o[m][2] *= ca; o[m][3] *= cb;
                    }
                }
                // probabilities carry the factor 2^kPExp (so do l_run and zacc; removed at the end)
                float pr[4];
                {
                    const float2 a01 = __fadd2_rn(make_float2(lg[0], lg[1]), make_float2(-m_off, -m_off));
                    const float2 a23 = __fadd2_rn(make_float2(lg[2], lg[3]), make_float2(-m_off, -m_off));
                    pr[0] = ex2(a01.x); pr[1] = ex2(a01.y); pr[2] = ex2(a23.x); pr[3] = ex2(a23.y);
                }
                l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);
                // ---- scale and zero rows of the lane's four tokens: one vector load per token and array
                float sf[4][G8], zf[4][G8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int toff = (e & 1) + 8 * (e >> 1);
                    load_halves<G8>(reinterpret_cast<const __half*>(stg + o_scl + toff * G8 * 2), sf[e]);
                    load_halves<G8>(reinterpret_cast<const __half*>(stg + o_zer + toff * G8 * 2), zf[e]);
                }
                // ---- zero term on FMAs: zacc[g] += p * z
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (G8 % 2 == 0) {
#pragma unroll
                        for (int g = 0; g < G8; g += 2) {
                            const float2 t = __ffma2_rn(make_float2(pr[e], pr[e]), make_float2(zf[e][g], zf[e][g + 1]),
                                                        make_float2(zacc[g], zacc[g + 1]));
                            zacc[g] = t.x;
                            zacc[g + 1] = t.y;
                        }
                    } else {
#pragma unroll
                        for (int g = 0; g < G8; ++g) zacc[g] = fmaf(pr[e], zf[e][g], zacc[g]);
                    }
                }
                // ---- values: A = codes (exact bf16), B = hi/lo of p * scale; per 32-column slice
                const uint8_t* vch = stg + o_val;
                uint32_t bh0 = 0, bh1 = 0, bl0 = 0, bl1 = 0;
#pragma unroll
                for (int sl = 0; sl < NSL; ++sl) {
                    const int g = (32 * sl) / VG;
                    if (sl == 0 || (32 * sl) % VG == 0) {
                        const float2 x01 = __fmul2_rn(make_float2(pr[0], pr[1]), make_float2(sf[0][g], sf[1][g]));
                        const float2 x23 = __fmul2_rn(make_float2(pr[2], pr[3]), make_float2(sf[2][g], sf[3][g]));
                        split_bf16(x01, bh0, bl0);
                        split_bf16(x23, bh1, bl1);
                    }
                    uint32_t f[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) f[e] = vfield<VB>(vch + ((e & 1) + 8 * (e >> 1)) * C::kVRow, sl, gid);
#pragma unroll
                    for (int hm = 0; hm < 2; ++hm) {
                        uint4 a;
                        if constexpr (VB == 8) {
                            const uint32_t s0 = 0x4400u + 0x1111u * (2 * hm), s1 = s0 + 0x1111u;
                            a.x = __byte_perm(f[0], f[1], s0) & 0x00FF00FFu;
                            a.y = __byte_perm(f[0], f[1], s1) & 0x00FF00FFu;
                            a.z = __byte_perm(f[2], f[3], s0) & 0x00FF00FFu;
                            a.w = __byte_perm(f[2], f[3], s1) & 0x00FF00FFu;
                        } else {
                            const uint32_t p01 = __byte_perm(f[0], f[1], 0x5410), p23 = __byte_perm(f[2], f[3], 0x5410);
                            a.x = vcode_sel<VB>(p01, 2 * hm);
                            a.y = vcode_sel<VB>(p01, 2 * hm + 1);
                            a.z = vcode_sel<VB>(p23, 2 * hm);
                            a.w = vcode_sel<VB>(p23, 2 * hm + 1);
                        }
                        mma_bf16(o[2 * sl + hm], a, bh0, bh1);
                        mma_bf16(o[2 * sl + hm], a, bl0, bl1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(b_empty + 8 * s);
        }

        // ------------------------------------------------------------------ per-warp finalisation
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
#pragma unroll
        for (int g = 0; g < G8; ++g) {
            zacc[g] += __shfl_xor_sync(0xffffffffu, zacc[g], 1);
            zacc[g] += __shfl_xor_sync(0xffffffffu, zacc[g], 2);
        }
        constexpr float kUnP = 1.0f / static_cast<float>(1ull << 40) / static_cast<float>(1ull << 40);  // 2^-kPExp
        float* zs = reinterpret_cast<float*>(smem + C::kZsOff) + warp * 8 * G8;
        if (tig == 0) {
#pragma unroll
            for (int g = 0; g < G8; ++g) zs[gid * G8 + g] = zacc[g] * kUnP;
        }
        // the stage ring is free once every consumer is past its last stage
        named_bar_sync(1, 32 * C::kWarps);
        float* comb = reinterpret_cast<float*>(smem);          // [warp][16 + 8D]
        float* mine = comb + warp * C::kPartFloats;
        if (tig == 0) {
            mine[gid] = m_run;
            mine[8 + gid] = l_run * kUnP;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                // row r = gid + 8 (e / 2) of m-tile m is value column 32 (m / 2) + 4 gid + pos, code position
                // pos = 2 (m % 2) + e / 2; column n = 2 tig + e % 2 is the head
                const int pos = 2 * (m & 1) + (e >> 1);
                const int col = 32 * (m >> 1) + 4 * gid + pos;
                const int hd = 2 * tig + (e & 1);
                // codes entered as code * 2^(scale + -133), probabilities as p * 2^kPExp
                const float unit = __int_as_float((127 + 133 - kPExp - vcode_scale_log2<VB>(pos)) << 23);
                mine[16 + hd * D + col] = o[m][e] * unit + zs[hd * G8 + col / VG];
            }
        }
        named_bar_sync(1, 32 * C::kWarps);
        // ------------------------------------------------------------------ merge the four warps
        const int tid = threadIdx.x;
        float* part = p.partials +
                      ((static_cast<int64_t>(b) * p.num_kv_heads + h) * p.num_parts + split) * C::kPartFloats;
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
            if (p.num_parts == 1) {
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
        // the merge grid (launched as a programmatic dependent) may start; it waits for this grid to finish
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
}

// Attention logits of the compressed path, for score-fidelity measurements: s[b][hq][t] = scale * n_t *
// <Pi_op q, c_op[idx_t]> (natural-log units) for t < len, -inf for len <= t < score_len.  Grid
// (ceil(chunks / 4), H_kv, B), 4 warps, one 16-token chunk each; the score contraction is the split kernel's
// (query fragments from attend_prep_kernel, code pairs from a per-bank replicated table, mma.sync).
template <int D, int KB>
__global__ void __launch_bounds__(128) attend_scores_kernel(const AttendParams p, float* __restrict__ scores,
                                                            int64_t score_len) {
    constexpr int KS = D / 16;
    constexpr int kKRow = D * KB / 8;
    constexpr int kQuarterHalves = D * KB / 4 / 16;
    constexpr int kQuarterWords = (kQuarterHalves + 1) / 2 + 1;
    constexpr int kPairs = key_table_entries<KB>();
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t lut_addr = (smem_u32(smem) + kPairs * 128 - 1) & ~static_cast<uint32_t>(kPairs * 128 - 1);
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + (lut_addr - smem_u32(smem)));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int h = blockIdx.y, b = blockIdx.z;
    const int G = p.group;
    fill_replicated(lut, p.pair_lut, kPairs);
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint4* qf = p.qfrag + (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.qfrag_stride;
    const float unpre = __ldcg(reinterpret_cast<const float*>(qf + KS * 32) + gid);
    const int64_t T = attend_seq_len(p, b);
    const int64_t chunk = static_cast<int64_t>(blockIdx.x) * 4 + warp;
    if (chunk * 16 >= score_len) return;
    // this lane's quarter of the key rows of tokens 8 nt + gid (zero past the sequence)
    uint32_t w[2][kQuarterWords];
    float nrm[2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int64_t tk = chunk * 16 + 8 * nt + gid;
#pragma unroll
        for (int i = 0; i < kQuarterWords; ++i) w[nt][i] = 0u;
        nrm[nt] = 0.f;
        if (tk < T) {
            const int64_t row = p.block_table
                ? (static_cast<int64_t>(p.block_table[static_cast<int64_t>(b) * p.max_blocks + tk / 16]) * p.num_kv_heads + h) * 16 + tk % 16
                : (static_cast<int64_t>(b) * p.num_kv_heads + h) * p.max_seq_len + tk;
            const uint16_t* k16 = reinterpret_cast<const uint16_t*>(p.k_packed + row * kKRow) + tig * kQuarterHalves;
#pragma unroll
            for (int i = 0; i < kQuarterWords; ++i) {
                const uint32_t lo16 = (2 * i < kQuarterHalves) ? k16[2 * i] : 0u;
                const uint32_t hi16 = (2 * i + 1 < kQuarterHalves) ? k16[2 * i + 1] : 0u;
                w[nt][i] = lo16 | (hi16 << 16);
            }
            nrm[nt] = p.k_norms[row];
        }
    }
    const uint32_t lane_addr = lut_addr + 4u * lane;
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        const uint4 a = __ldcg(qf + ks * 32 + lane);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            mma_f16(sc[nt], a, key_b_reg<KB, true>(w[nt], 4 * ks, lane_addr),
                    key_b_reg<KB, true>(w[nt], 4 * ks + 2, lane_addr));
        }
    }
    // C columns 2 tig, 2 tig + 1 of n-tile nt are tokens 8 nt + 2 tig (+1), whose norms sit in lanes 4 (2 tig + k)
    float tn[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int k = 0; k < 2; ++k) tn[nt][k] = __shfl_sync(0xffffffffu, nrm[nt], 4 * (2 * tig + k));
    }
    if (gid < G) {
        float* srow = scores + (static_cast<int64_t>(b) * p.num_q_heads + static_cast<int64_t>(h) * G + gid) * score_len;
        constexpr float kLn2 = 0.69314718055994530942f;   // the fragments carry scale * log2(e)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int64_t t = chunk * 16 + 8 * nt + 2 * tig + k;
                if (t < score_len)
                    srow[t] = (t < T) ? (sc[nt][k] + sc[nt][k + 2]) * unpre * tn[nt][k] * kLn2 : -INFINITY;
            }
        }
    }
}

// Split-K merge: out[b][h*G+g][:] = sum_s O_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), M = max_s m_s.
// Grid (G * D/32, H_kv, B): each CTA merges 32 columns of one (query head, kv head, sequence), so the partials
// are read by four times as many SMs as with one CTA per head.  Slice k of the CTA's threads folds splits
// k, k + kSlices, ... with every load issued before the first is used (one round trip per batch); the slices
// are then combined in shared memory the same way.
constexpr int kMergeThreads = 256;
constexpr int kMergeCols = 32;
constexpr int kMaxSplits = 256;

template <int D>
__global__ void __launch_bounds__(kMergeThreads) attend_merge_kernel(const AttendParams p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int kPart = 16 + 8 * D;
    constexpr int kCS = D / kMergeCols;
    constexpr int kSlices = kMergeThreads / kMergeCols;
    constexpr int kBatch = 12;                           // splits per slice per round of loads
    __shared__ float s_o[kSlices][kMergeCols];
    __shared__ float s_ml[kSlices][2];
    const int g = blockIdx.x / kCS, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int lc = tid % kMergeCols, slice = tid / kMergeCols;
    const int col = (blockIdx.x % kCS) * kMergeCols + lc;
    const int S = p.num_parts;
    const float* base = p.partials + (static_cast<int64_t>(b) * p.num_kv_heads + h) * S * kPart;
    float M = -INFINITY, L = 0.f, O = 0.f;
    for (int s0 = slice; s0 < S; s0 += kSlices * kBatch) {
        float mv[kBatch], lv[kBatch], ov[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int sp = s0 + k * kSlices;
            const float* ps = base + static_cast<int64_t>(sp < S ? sp : 0) * kPart;
            mv[k] = (sp < S) ? __ldcg(ps + g) : -INFINITY;
            lv[k] = __ldcg(ps + 8 + g);
            ov[k] = __ldcg(ps + 16 + g * D + col);
        }
        float Mn = M;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) Mn = fmaxf(Mn, mv[k]);
        const float Mu = (Mn == -INFINITY) ? 0.f : Mn;
        const float c = exp2f(M - Mu);
        L *= c;
        O *= c;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const float f = exp2f(mv[k] - Mu);                // 0 for the padding entries
            L = fmaf(lv[k], f, L);
            O = fmaf(ov[k], f, O);
        }
        M = Mn;
    }
    s_o[slice][lc] = O;
    if (lc == 0) {
        s_ml[slice][0] = M;
        s_ml[slice][1] = L;
    }
    __syncthreads();
    if (slice == 0) {
        float Mt = s_ml[0][0];
#pragma unroll
        for (int k = 1; k < kSlices; ++k) Mt = fmaxf(Mt, s_ml[k][0]);
        const float Mu = (Mt == -INFINITY) ? 0.f : Mt;
        float Lt = 0.f, Ot = 0.f;
#pragma unroll
        for (int k = 0; k < kSlices; ++k) {
            const float f = exp2f(s_ml[k][0] - Mu);
            Lt = fmaf(s_ml[k][1], f, Lt);
            Ot = fmaf(s_o[k][lc], f, Ot);
        }
        p.out[(static_cast<int64_t>(b) * p.num_q_heads + static_cast<int64_t>(h) * p.group + g) * D + col] =
            (Lt > 0.f) ? Ot / Lt : 0.f;
    }
}

}  // namespace dev
}  // namespace tq
