// Weight preparation: N:M magnitude mask, per-row absmean scale over the kept
// weights, ternarisation and 2-bit packing, fused in one pass per row.
//
// Operator: Sparse-BitNet Guide: 1.58-Bit LLMs Meet 2:4 Sparsity, "Mathematical
// Formulation of Sparse-BitLinear" (mask equation, joint sparse-ternary
// equation); per-row absmean from the halo-sparse-bitnet-3:4-500m card,
// "Recipe"; code table 00 = 0, 01 = +1, 10 = -1 from its "Packed vs raw".
//
// TPR threads share a row (256 / TPR rows per block); each thread owns up to
// two 16-weight chunks, read once as 16-byte loads and kept in registers.
// Pass 1 builds the keep-mask of every group and adds the kept |w| exactly
// into a register window anchored at the row's largest kept magnitude (see
// kWindow); after a block-wide reduction of the row sums, pass 2 ternarises
// the registers against the row scale and writes one 32-bit word of codes and
// 16 mask bits per chunk.  Rows longer than 512 chunks (K > 8192) use a
// warp-per-row variant that reads the row twice and sums in shared-memory limbs.
//
// Exact sum: a finite float |w| = m * 2^(p - 149) with a 24-bit integer m and
// 0 <= p <= 253, so the row sum is an integer in units of 2^-149 below 2^300.
// Each lane keeps it in ten 32-bit limbs held in 64-bit shared-memory words
// (carries are resolved once, at the end), which makes the sum independent of
// the order of additions; the total is rounded once to double.
#include "sbl_common.cuh"

namespace sbl {

constexpr int kPrepWarps = 8;
constexpr int kLimbs = 10;

__device__ __forceinline__ void exact_add(unsigned long long* limb_col, uint32_t abs_bits) {
    const uint32_t e = abs_bits >> 23;
    const uint32_t m24 = (abs_bits & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    const uint32_t p = e ? e - 1u : 0u;
    const uint32_t li = p >> 5;
    const unsigned long long v = static_cast<unsigned long long>(m24) << (p & 31u);
    limb_col[li * 32] += v & 0xFFFFFFFFull;
    limb_col[(li + 1) * 32] += v >> 32;
}

// Round the 320-bit integer w[0..9] (32-bit limbs, units of 2^-149) to double.
__device__ double limbs_to_double(const uint32_t (&w)[kLimbs]) {
    int h = -1;
#pragma unroll
    for (int i = kLimbs - 1; i >= 0; --i)
        if (h < 0 && w[i] != 0u) h = i;
    const double two_m149 = 1.4012984643248170709e-45;  // 2^-149, exact
    if (h < 0) return 0.0;
    if (h <= 1) {
        const unsigned long long x = (static_cast<unsigned long long>(w[1]) << 32) | w[0];
        return __ull2double_rn(x) * two_m149;
    }
    const int lz = __clz(w[h]);
    unsigned long long top;
    uint32_t dropped;
    if (lz == 0) {
        top = (static_cast<unsigned long long>(w[h]) << 32) | w[h - 1];
        dropped = w[h - 2];
    } else {
        top = (static_cast<unsigned long long>(w[h]) << (32 + lz)) |
              (static_cast<unsigned long long>(w[h - 1]) << lz) | (w[h - 2] >> (32 - lz));
        dropped = w[h - 2] & ((1u << (32 - lz)) - 1u);
    }
    for (int i = 0; i < h - 2; ++i) dropped |= w[i];
    top |= (dropped != 0u) ? 1ull : 0ull;  // sticky bit: below the rounding position
    const int e2 = 32 * h - 32 - lz - 149;  // weight of bit 0 of `top`
    const double scale = __longlong_as_double(static_cast<long long>(1023 + e2) << 52);
    return __ull2double_rn(top) * scale;
}

// keep[i] for the M weights of one group: rank by magnitude, ties to the lower index.
template <int M>
__device__ __forceinline__ uint32_t group_keep_bits(const uint32_t* a, int n) {
    int rank[M];
#pragma unroll
    for (int j = 0; j < M; ++j) rank[j] = 0;
#pragma unroll
    for (int i = 0; i < M; ++i)
#pragma unroll
        for (int j = i + 1; j < M; ++j) {
            if (a[i] >= a[j]) ++rank[j];
            else ++rank[i];
        }
    uint32_t bits = 0;
#pragma unroll
    for (int j = 0; j < M; ++j) bits |= (rank[j] < n ? 1u : 0u) << j;
    return bits;
}

template <int M>
__device__ __forceinline__ uint32_t chunk_keep_bits(const uint32_t (&a)[16], int n) {
    uint32_t bits = 0;
#pragma unroll
    for (int g = 0; g < 16 / M; ++g) bits |= group_keep_bits<M>(a + g * M, n) << (g * M);
    return bits;
}

__device__ __forceinline__ void load_chunk(const float* p, uint32_t (&bits)[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = ldg_nc(p + 4 * q);
        bits[4 * q + 0] = v.x;
        bits[4 * q + 1] = v.y;
        bits[4 * q + 2] = v.z;
        bits[4 * q + 3] = v.w;
    }
}

template <int M>
__global__ void __launch_bounds__(kPrepWarps * 32) prep_kernel(const float* __restrict__ W, long long O, long long K,
                                                               int n, uint8_t* __restrict__ packed,
                                                               float* __restrict__ row_scale,
                                                               uint8_t* __restrict__ mask_bits, unsigned* status) {
    __shared__ unsigned long long limbs[kPrepWarps][kLimbs][32];
    __shared__ unsigned long long totals[kPrepWarps][kLimbs];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * kPrepWarps + warp;
    if (row >= O) return;  // whole warps leave together; no block barrier below

    const float* wr = W + row * K;
    const int nchunks = static_cast<int>(K >> 4);
    unsigned long long* my = &limbs[warp][0][lane];
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) my[l * 32] = 0ull;

    bool bad = false;
    for (int c = lane; c < nchunks; c += 32) {
        uint32_t a[16];
        load_chunk(wr + 16 * c, a);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            a[i] &= 0x7FFFFFFFu;
            bad |= a[i] >= 0x7F800000u;
        }
        const uint32_t keep = chunk_keep_bits<M>(a, n);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (keep & (1u << i)) exact_add(my, a[i]);
    }
    __syncwarp();
    if (lane < kLimbs) {
        unsigned long long s = 0;
        for (int i = 0; i < 32; ++i) s += limbs[warp][lane][i];
        totals[warp][lane] = s;
    }
    __syncwarp();

    float scale = 0.f;
    if (lane == 0) {
        uint32_t w[kLimbs];
        unsigned long long carry = 0;
#pragma unroll
        for (int i = 0; i < kLimbs; ++i) {
            const unsigned long long t = totals[warp][i] + carry;
            w[i] = static_cast<uint32_t>(t);
            carry = t >> 32;
        }
        const double sum = limbs_to_double(w);
        const double kept = static_cast<double>((K / M) * n);
        scale = fmaxf(__double2float_rn(__ddiv_rn(sum, kept)), 1e-5f);
        row_scale[row] = scale;
    }
    scale = __shfl_sync(0xFFFFFFFFu, scale, 0);
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_status(status, kStatusNonfinite);

    const uint32_t half_bits = __float_as_uint(0.5f * scale);  // exact: scale >= 1e-5 is normal
    uint32_t* prow = reinterpret_cast<uint32_t*>(packed + row * (K >> 2));
    uint16_t* mrow = mask_bits ? reinterpret_cast<uint16_t*>(mask_bits + row * (K >> 3)) : nullptr;
    for (int c = lane; c < nchunks; c += 32) {
        uint32_t raw[16], a[16];
        load_chunk(wr + 16 * c, raw);
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = raw[i] & 0x7FFFFFFFu;
        const uint32_t keep = chunk_keep_bits<M>(a, n);
        uint32_t codes = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            // round(w / scale) != 0  <=>  |w| / scale > 1/2  <=>  |w| > scale / 2 (exact compare)
            const bool nz = ((keep >> i) & 1u) && (a[i] > half_bits);
            const uint32_t code = nz ? ((raw[i] >> 31) ? 2u : 1u) : 0u;
            codes |= code << (2 * i);
        }
        prow[c] = codes;
        if (mrow) mrow[c] = static_cast<uint16_t>(keep);
    }
}

constexpr int kPrepThreads = 256;

// Exact row sums in registers.  With p_max the largest exponent index among the
// row's kept magnitudes (|w| = m * 2^(p - 149), m < 2^24), every kept value
// with p >= base = p_max - 96 is added exactly into a 128-bit per-thread
// accumulator in units of 2^(base - 149) (a value is below 2^120 there and a
// thread adds at most 32 of them); smaller values only set a sticky flag.
// Their total is below 2^24 * 2^base, at least 2^40 times smaller than the
// rounding position of a double holding the sum (which is >= 2^(p_max + 23)),
// so the 192-bit row total plus the sticky flag rounds to the same double as
// the exact sum.
constexpr int kWindow = 96;

__device__ __forceinline__ void add128(unsigned long long& w0, unsigned long long& w1, unsigned long long a0,
                                       unsigned long long a1) {
    asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, %3;" : "+l"(w0), "+l"(w1) : "l"(a0), "l"(a1));
}

__device__ __forceinline__ void add192(unsigned long long (&w)[3], const unsigned long long (&a)[3]) {
    asm("add.cc.u64 %0, %0, %3;\n\taddc.cc.u64 %1, %1, %4;\n\taddc.u64 %2, %2, %5;"
        : "+l"(w[0]), "+l"(w[1]), "+l"(w[2])
        : "l"(a[0]), "l"(a[1]), "l"(a[2]));
}

// Round w[0..2] * 2^(base - 149) (+ a sticky remainder) to double.
__device__ double window_to_double(const unsigned long long (&w)[3], bool sticky, int base) {
    int h = 2;
    while (h >= 0 && w[h] == 0ull) --h;
    if (h < 0) return 0.0;  // sticky alone cannot happen: dropped values are nonzero only next to larger ones
    const int lz = __clzll(w[h]);
    unsigned long long top = w[h] << lz;
    unsigned long long rest = 0;  // bits below `top`
    if (h >= 1) {
        if (lz) top |= w[h - 1] >> (64 - lz);
        rest = w[h - 1] << lz;
        if (lz == 0) rest = w[h - 1];
        if (h == 2) rest |= w[0];
    }
    if (rest || sticky) top |= 1ull;  // sticky bit: below the rounding position
    const int e2 = 64 * h + (64 - lz) - 64 + base - 149;  // weight of bit 0 of `top`
    const double scale = __longlong_as_double(static_cast<long long>(1023 + e2) << 52);
    return __ull2double_rn(top) * scale;
}

template <int M, int TPR>
__global__ void __launch_bounds__(kPrepThreads) prep_kernel_rr(const float* __restrict__ W, long long O,
                                                               long long K, int n, uint8_t* __restrict__ packed,
                                                               float* __restrict__ row_scale,
                                                               uint8_t* __restrict__ mask_bits, unsigned* status) {
    constexpr int RPB = kPrepThreads / TPR;  // rows per block
    constexpr int CPT = 2;                   // chunks per thread
    constexpr int WPR = TPR / 32;            // warps per row
    __shared__ uint32_t wmax[kPrepThreads / 32];
    __shared__ unsigned long long wsum[kPrepThreads / 32][3];
    __shared__ uint32_t wsticky[kPrepThreads / 32];
    __shared__ float scales[RPB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = threadIdx.x / TPR, tr = threadIdx.x % TPR;
    const long long row = static_cast<long long>(blockIdx.x) * RPB + sub;
    const bool valid = row < O;
    const int nchunks = static_cast<int>(K >> 4);
    const float* wr = W + (valid ? row : 0) * K;

    uint32_t raw[CPT][16];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = tr + TPR * j;
        if (valid && c < nchunks) load_chunk(wr + 16 * c, raw[j]);
        else
#pragma unroll
            for (int i = 0; i < 16; ++i) raw[j][i] = 0u;
    }

    // keep-masks, non-finite check and the largest kept magnitude of the row
    bool bad = false;
    uint32_t keep[CPT];
    uint32_t mx = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        uint32_t a[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            a[i] = raw[j][i] & 0x7FFFFFFFu;
            bad |= a[i] >= 0x7F800000u;
        }
        keep[j] = chunk_keep_bits<M>(a, n);
        const int c = tr + TPR * j;
        if (!(valid && c < nchunks)) keep[j] = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (keep[j] & (1u << i)) mx = max(mx, a[i]);
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) wmax[warp] = mx;
    if (__syncthreads_or(bad ? 1 : 0) && threadIdx.x == 0) raise_status(status, kStatusNonfinite);
#pragma unroll
    for (int w = 0; w < WPR; ++w) mx = max(mx, wmax[sub * WPR + w]);
    const int emax = static_cast<int>(mx >> 23);
    const int base = (emax ? emax - 1 : 0) - kWindow;

    // exact accumulation of the kept magnitudes
    unsigned long long w0 = 0, w1 = 0;
    uint32_t sticky = 0;
#pragma unroll
    for (int j = 0; j < CPT; ++j)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (!(keep[j] & (1u << i))) continue;
            const uint32_t a = raw[j][i] & 0x7FFFFFFFu;
            const uint32_t e = a >> 23;
            const uint32_t m24 = (a & 0x7FFFFFu) | (e ? 0x800000u : 0u);
            const int sh = (e ? static_cast<int>(e) - 1 : 0) - base;  // <= kWindow
            if (sh < 0) {
                sticky |= m24;
            } else {
                const int bit = sh & 63;
                const unsigned long long v = static_cast<unsigned long long>(m24) << bit;
                const unsigned long long hi = bit > 40 ? static_cast<unsigned long long>(m24) >> (64 - bit) : 0ull;
                if (sh < 64) add128(w0, w1, v, hi);
                else add128(w0, w1, 0ull, v);
            }
        }

    // row total: warp butterfly on 192 bits, then the row's warps
    unsigned long long t[3] = {w0, w1, 0ull};
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const unsigned long long o[3] = {__shfl_xor_sync(0xFFFFFFFFu, t[0], off),
                                         __shfl_xor_sync(0xFFFFFFFFu, t[1], off),
                                         __shfl_xor_sync(0xFFFFFFFFu, t[2], off)};
        add192(t, o);
    }
    sticky = __reduce_or_sync(0xFFFFFFFFu, sticky);
    if (lane == 0) {
        wsum[warp][0] = t[0];
        wsum[warp][1] = t[1];
        wsum[warp][2] = t[2];
        wsticky[warp] = sticky;
    }
    __syncthreads();
    if (tr == 0) {
        unsigned long long tot[3] = {0ull, 0ull, 0ull};
        uint32_t st = 0;
#pragma unroll
        for (int w = 0; w < WPR; ++w) {
            const unsigned long long o[3] = {wsum[sub * WPR + w][0], wsum[sub * WPR + w][1], wsum[sub * WPR + w][2]};
            add192(tot, o);
            st |= wsticky[sub * WPR + w];
        }
        const double sum = window_to_double(tot, st != 0, base);
        const double kept = static_cast<double>((K / M) * n);
        const float sc = fmaxf(__double2float_rn(__ddiv_rn(sum, kept)), 1e-5f);
        scales[sub] = sc;
        if (valid) row_scale[row] = sc;
    }
    __syncthreads();
    if (!valid) return;
    const uint32_t half_bits = __float_as_uint(0.5f * scales[sub]);  // exact: scale >= 1e-5 is normal
    uint32_t* prow = reinterpret_cast<uint32_t*>(packed + row * (K >> 2));
    uint16_t* mrow = mask_bits ? reinterpret_cast<uint16_t*>(mask_bits + row * (K >> 3)) : nullptr;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = tr + TPR * j;
        if (c >= nchunks) continue;
        uint32_t codes = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            // round(w / scale) != 0  <=>  |w| / scale > 1/2  <=>  |w| > scale / 2 (exact compare)
            const bool nz = ((keep[j] >> i) & 1u) && ((raw[j][i] & 0x7FFFFFFFu) > half_bits);
            codes |= (nz ? ((raw[j][i] >> 31) ? 2u : 1u) : 0u) << (2 * i);
        }
        prow[c] = codes;
        if (mrow) mrow[c] = static_cast<uint16_t>(keep[j]);
    }
}

template <int M, int TPR>
static void launch_prep_rr(const float* W, long long O, long long K, int n, uint8_t* packed, float* row_scale,
                           uint8_t* mask_bits, unsigned* status, cudaStream_t stream) {
    constexpr int RPB = kPrepThreads / TPR;
    const unsigned blocks = static_cast<unsigned>((O + RPB - 1) / RPB);
    prep_kernel_rr<M, TPR><<<blocks, kPrepThreads, 0, stream>>>(W, O, K, n, packed, row_scale, mask_bits, status);
}

template <int M>
static void launch_prep_m(const float* W, long long O, long long K, int n, uint8_t* packed, float* row_scale,
                          uint8_t* mask_bits, unsigned* status, cudaStream_t stream) {
    const long long nchunks = K >> 4;
    if (nchunks <= 64) launch_prep_rr<M, 32>(W, O, K, n, packed, row_scale, mask_bits, status, stream);
    else if (nchunks <= 128) launch_prep_rr<M, 64>(W, O, K, n, packed, row_scale, mask_bits, status, stream);
    else if (nchunks <= 256) launch_prep_rr<M, 128>(W, O, K, n, packed, row_scale, mask_bits, status, stream);
    else if (nchunks <= 512) launch_prep_rr<M, 256>(W, O, K, n, packed, row_scale, mask_bits, status, stream);
    else {
        const unsigned blocks = static_cast<unsigned>((O + kPrepWarps - 1) / kPrepWarps);
        prep_kernel<M><<<blocks, kPrepWarps * 32, 0, stream>>>(W, O, K, n, packed, row_scale, mask_bits, status);
    }
}

cudaError_t launch_prep(const float* W, long long O, long long K, int n, int m, uint8_t* packed, float* row_scale,
                        uint8_t* mask_bits, unsigned* status, cudaStream_t stream) {
    if (m == 4) launch_prep_m<4>(W, O, K, n, packed, row_scale, mask_bits, status, stream);
    else launch_prep_m<8>(W, O, K, n, packed, row_scale, mask_bits, status, stream);
    return cudaGetLastError();
}

}  // namespace sbl
