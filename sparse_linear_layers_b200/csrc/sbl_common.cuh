// Shared device helpers of the Sparse-BitLinear kernels (sm_100a only).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sbl {

// Launch as a programmatic dependent of the previous kernel on the stream:
// the kernel may start (and run its prologue) while its predecessor drains,
// and must execute griddepcontrol.wait before reading anything the
// predecessor writes.
template <typename Kern, typename... Args>
inline cudaError_t pdl_launch(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Bits of the per-device status word (see sbl_device_status in sbl.h).
constexpr unsigned kStatusNonfinite = 1u;
constexpr unsigned kStatusTimeout = 2u;
constexpr unsigned kStatusInvalid = 4u;  // input data the kernel cannot represent (not 2:4 where 2:4 is required)

// Upper bound of any pipeline wait: a healthy wait is microseconds; after this
// the kernel records a timeout and winds down instead of spinning forever.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void raise_status(unsigned* status, unsigned bit) {
    atomicOr(status, bit);
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false when the
// CTA-wide abort flag is set or the time limit passes (the caller then winds
// down); never spins without limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 0u) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > kWaitLimitNs) return false;
        }
    }
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded spin on the non-blocking test: for single-thread roles (MMA issue,
// TMA producer) whose reaction time after a phase completes matters.
__device__ __forceinline__ bool mbar_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_test_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 255u) == 0u) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > kWaitLimitNs) return false;
        }
    }
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- loads
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// dp4a with unsigned bytes in a and signed bytes in b.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Byte permute, PTX default mode (selector nibble bit 3 replicates the sign bit).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Expand one 32-bit word of 2-bit codes (16 weights, weight i at bits 2i..2i+1,
// 00 = 0, 01 = +1, 10 = -1) into four int8x4 words.  Word j holds the weights
// 4b + j (b = 0..3) in byte b, i.e. the 16 weights come out in the order
// 0,4,8,12, 1,5,9,13, 2,6,10,14, 3,7,11,15; activations are stored in the same
// order ("interleaved") so dot products need no further shuffling.
__device__ __forceinline__ void expand_codes(uint32_t w, uint32_t (&out)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t hi_at_msb = (j == 3) ? w : (w << (6 - 2 * j));    // bit 2j+1 of each byte -> bit 7
        const uint32_t neg = prmt(hi_at_msb, 0u, 0xBA98u);              // 0xFF where the code is 10
        const uint32_t lo = (j == 0 ? w : (w >> (2 * j))) & 0x01010101u; // 0x01 where the code is 01
        out[j] = neg | lo;
    }
}

// Expand one 32-bit code word into four int8x4 words, pairing order: word 0
// holds weights 0, 2, 4, 6, word 1 weights 1, 3, 5, 7, word 2 weights 8, 10,
// 12, 14 and word 3 weights 9, 11, 13, 15 (byte b = the b-th of each list).
// Each is one byte permute whose selector nibbles are the 2-bit codes
// themselves, from a table whose bytes 0, 1, 2 are the values 0, +1, -1 of
// codes 00, 01, 10.  Activations are stored in the same order
// (quant_block16_pairs) so dot products need no further shuffling.
constexpr uint32_t kTernaryBytes = 0x00FF0100u;
__device__ __forceinline__ void expand_pairs(uint32_t w, uint32_t (&e)[4]) {
    const uint32_t lo = w & 0x33333333u;           // codes of the even weights, one per nibble
    const uint32_t hi = (w >> 2) & 0x33333333u;    // codes of the odd weights
    e[0] = prmt(kTernaryBytes, 0u, lo);
    e[1] = prmt(kTernaryBytes, 0u, hi);
    e[2] = prmt(kTernaryBytes, 0u, lo >> 16);
    e[3] = prmt(kTernaryBytes, 0u, hi >> 16);
}

// ---------------------------------------------------------------- activation quantisation
// round_half_even(x * s) for an activation x (as float) and its token's
// s = 127 / max|x|, returned as the bit pattern of x * s + 1.5 * 2^23.  The
// product is rounded to float first, as in the definition; adding 1.5 * 2^23
// then rounds it to an integer (IEEE round to nearest even) that lands in the
// low mantissa bits, so the low byte is the int8 two's-complement code.  For
// finite x, |x * s| <= 127 (s is the correctly rounded 127 / max|x| and
// |x| <= max|x|), so the clamp to [-128, 127] never acts and is not applied.
__device__ __forceinline__ uint32_t quant_code_bits(float x, float s) {
    return __float_as_uint(__fadd_rn(__fmul_rn(x, s), 12582912.0f));
}

// Low bytes of four code words into one int8x4 word (a in byte 0).
__device__ __forceinline__ uint32_t pack_codes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return prmt(prmt(a, b, 0x0040u), prmt(c, d, 0x0040u), 0x5410u);
}

// Codes of the 16 activations held as eight bf16 pairs (element 2i in the low
// half of word i, 2i + 1 in the high half).
__device__ __forceinline__ void quant_codes16(const uint4& u0, const uint4& u1, float s, uint32_t (&q)[16]) {
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        q[2 * i] = quant_code_bits(__uint_as_float(w[i] << 16), s);
        q[2 * i + 1] = quant_code_bits(__uint_as_float(w[i] & 0xFFFF0000u), s);
    }
}

__device__ __forceinline__ uint32_t absmax8(const uint4& u, uint32_t mx) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        mx = max(mx, w[i] & 0x7FFFu);
        mx = max(mx, (w[i] >> 16) & 0x7FFFu);
    }
    return mx;
}


// Quantise 16 consecutive activations (two 16-byte vectors of bf16) and return
// them as four int8x4 words, either in column order or interleaved (byte
// 4j + b <- element 4b + j, the order of expand_codes()).
template <bool INTERLEAVED>
__device__ __forceinline__ uint4 quant_block16(const uint4& u0, const uint4& u1, float s) {
    uint32_t q[16];
    quant_codes16(u0, u1, s, q);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (INTERLEAVED)
            o[j] = pack_codes(q[j], q[4 + j], q[8 + j], q[12 + j]);
        else
            o[j] = pack_codes(q[4 * j], q[4 * j + 1], q[4 * j + 2], q[4 * j + 3]);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Quantise 16 consecutive activations into the pairing order of expand_pairs().
__device__ __forceinline__ uint4 quant_block16_pairs(const uint4& u0, const uint4& u1, float s) {
    uint32_t q[16];
    quant_codes16(u0, u1, s, q);
    return make_uint4(pack_codes(q[0], q[2], q[4], q[6]), pack_codes(q[1], q[3], q[5], q[7]),
                      pack_codes(q[8], q[10], q[12], q[14]), pack_codes(q[9], q[11], q[13], q[15]));
}

}  // namespace sbl
