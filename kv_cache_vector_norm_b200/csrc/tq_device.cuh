// Device helpers for sm_100a: mbarriers with bounded waits, TMA (tensor and bulk) copies, and the
// tcgen05 tensor-core / tensor-memory instructions, as inline PTX.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace tq {
namespace dev {

// Raised (OR-ed) by a kernel whose bounded wait expired; read by tq_read_device_flag().
__device__ unsigned int g_error_flag;

enum : unsigned { kFlagWaitTimeout = 1u };

// One bounded wait gives up after about a second at the B200's ~1.9 GHz SM clock.
constexpr long long kWaitLimitCycles = 1ll << 31;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void raise_flag(unsigned code) { atomicOr(&g_error_flag, code); }

// ------------------------------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase of `bar` with the given parity has completed.  Gives up after
// kWaitLimitCycles, raises the device flag and sets *abort (a shared-memory flag every role polls),
// returning false.  Also returns false at once if *abort is already set.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          long long limit = kWaitLimitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - start > limit) {
            *abort = 1;
            raise_flag(kFlagWaitTimeout);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag: used to drain copies or MMAs still in flight before a CTA
// releases shared or tensor memory, on the normal and the abort path alike.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, long long limit = kWaitLimitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - start > limit) {
            raise_flag(kFlagWaitTimeout);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// 2-D tensor store shared -> global in this thread's bulk group (x is the innermost coordinate; a box that
// reaches past the tensor's extent is clipped there).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}

// Untiled bulk copy global -> shared (both addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// 16-byte asynchronous global -> shared copy through L2 (both addresses 16-byte aligned).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued before has completed; the arrival does not count
// towards the pending count, so the barrier's expected count includes it.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Bulk (TMA, untiled) shared -> global stores in bulk groups of this thread.
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (fp16 or bf16 operands, fp32 accumulator).
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16: A is 128 rows (TMEM lanes) x 16 K-elements, two 16-bit
// elements per 32-bit column (8 columns from a_tmem).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives lane (quarter*32 + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp writes lane (quarter*32 + i).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand in the 128-byte-swizzled canonical layout:
// rows of 128 bytes (64 fp16), 8-row atoms of 1024 bytes stacked at a 1024-byte stride (SBO),
// 16-byte chunks of row r XOR-permuted by r % 8.  Advancing K by 16 fp16 inside the atom adds 32 bytes
// to the start address.  Fields: start>>4 [0,14), LBO>>4 [16,30) (unused by swizzled K-major, 1),
// SBO>>4 [32,46), version 1 [46,48), base offset 0 [49,52), layout SWIZZLE_128B = 2 [61,64).
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor of kind::f16 with fp16 A and B (K-major), fp32 D, shape M x N.
// Fields: D format [4,6) = 1 (F32); A format [7,10) = 0 (F16); B format [10,13) = 0 (F16);
// A/B major [15], [16] = 0 (K); N >> 3 at [17,23); M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int m, int n) {
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a 128-byte-swizzled region.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// --------------------------------------------------------------------------------- bit-field helpers

// OR value v (< 2^BITS) into the little-endian bitstream `w` at field j (compile-time after unrolling).
template <int BITS, int NW>
__device__ __forceinline__ void put_field(uint32_t (&w)[NW], int j, uint32_t v) {
    const int bit = j * BITS, wi = bit >> 5, sh = bit & 31;
    w[wi] |= v << sh;
    if (sh + BITS > 32) w[wi + 1] |= v >> (32 - sh);
}

// 32-bit load from a shared-space address (no memory clobber: callers order it after the barrier or wait
// that made the data visible, through the address's data dependence).
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Two 32-bit words from an 8-byte aligned shared-space address (same ordering rule as lds_u32).
__device__ __forceinline__ uint2 lds_u64(uint32_t addr) {
    uint2 v;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// Add value v (< 2^BITS) into field j of the zero-initialised bitstream `w` (fields do not overlap, so this is
// the same as OR-ing it in, as a shift-add).
template <int BITS, int NW>
__device__ __forceinline__ void add_field(uint32_t (&w)[NW], int j, uint32_t v) {
    const int bit = j * BITS, wi = bit >> 5, sh = bit & 31;
    w[wi] += v << sh;
    if (sh + BITS > 32) w[wi + 1] += v >> (32 - sh);
}

// acc + h * h for an fp16 h (given by its bits) with one rounding: h * h is exact in fp32
__device__ __forceinline__ float fma_f16_f32(uint16_t h, float acc) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %1, %2;" : "=f"(d) : "h"(h), "f"(acc));
    return d;
}

// A table replicated once per shared-memory bank (entry e of lane l at word 32 e + l) filled from `entries` words
// of global memory by all threads of the block: each entry is read once and written as eight 16-byte stores, so
// the fill costs one round trip to L2 per thread instead of one per word.
__device__ __forceinline__ void fill_replicated_by(uint32_t* dst, const uint32_t* __restrict__ src, int entries,
                                                   int tid, int nthreads) {
    for (int e = tid; e < entries; e += nthreads) {
        const uint32_t v = __ldg(src + e);
        uint4* d = reinterpret_cast<uint4*>(dst + 32 * e);
        const uint4 q = make_uint4(v, v, v, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) d[k] = q;
    }
}

__device__ __forceinline__ void fill_replicated(uint32_t* dst, const uint32_t* __restrict__ src, int entries) {
    for (int e = threadIdx.x; e < entries; e += blockDim.x) {
        const uint32_t v = __ldg(src + e);
        uint4* d = reinterpret_cast<uint4*>(dst + 32 * e);
        const uint4 q = make_uint4(v, v, v, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) d[k] = q;
    }
}

// Field of width W starting at bit `bit` of the little-endian bitstream `w`.
template <int W, int NW>
__device__ __forceinline__ uint32_t get_bits(const uint32_t (&w)[NW], int bit) {
    const int wi = bit >> 5, sh = bit & 31;
    uint32_t v = w[wi] >> sh;
    if (sh + W > 32) v |= w[wi + 1] << (32 - sh);
    return (W == 32) ? v : (v & ((1u << W) - 1u));
}

// The little-endian bitstream `w` shifted right by `bit` (-31 <= bit; bit + 32 <= 32 NW), low 32 bits.
template <int NW>
__device__ __forceinline__ uint32_t bits_shr(const uint32_t (&w)[NW], int bit) {
    if (bit < 0) return w[0] << (-bit);
    const int wi = bit >> 5, sh = bit & 31;
    if (sh == 0) return w[wi];
    return (wi + 1 < NW) ? __funnelshift_r(w[wi], w[wi + 1], sh) : (w[wi] >> sh);
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

// Load NW words with the widest vector loads NW allows: 16-byte loads when NW % 4 == 0 and 8-byte loads when
// NW is even, so `src` must be aligned to 16 or 8 bytes in those cases (4 otherwise).
template <int NW>
__device__ __forceinline__ void load_words(const uint8_t* src, uint32_t (&w)[NW]) {
    if constexpr (NW % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 4) {
            uint4 v = *reinterpret_cast<const uint4*>(src + 4 * i);
            w[i] = v.x; w[i + 1] = v.y; w[i + 2] = v.z; w[i + 3] = v.w;
        }
    } else if constexpr (NW % 2 == 0) {
#pragma unroll
        for (int i = 0; i < NW; i += 2) {
            uint2 v = *reinterpret_cast<const uint2*>(src + 4 * i);
            w[i] = v.x; w[i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = reinterpret_cast<const uint32_t*>(src)[i];
    }
}

// ------------------------------------------------------------------------------------- small helpers

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace dev
}  // namespace tq
