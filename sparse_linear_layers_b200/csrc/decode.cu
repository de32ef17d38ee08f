// Decode path: y = dequant(x_q . W_t^T) for a handful of tokens on CUDA cores.
//
// The integer product of the Sparse-BitNet Guide's linear-evaluation equation
// ("Mathematical Formulation of Sparse-BitLinear") for small T is a stream over
// the 2-bit weights (0.25 B per weight, read once), so it is bound by HBM
// bandwidth; the guide notes that memory bandwidth decides serving cost.
//
// Layout: a row of packed weights is K/4 bytes = CPR chunks of CW 32-bit words
// (16 CW weights; CW = 4 when K % 64 == 0 so rows are 16-byte aligned, else
// CW = 1).  L lanes share a row (32/L rows per warp, one row group per warp);
// lane li takes chunks li, li + L, ... in batches of NB chunks whose loads are
// all in flight together.
//
// The kernel is a programmatic dependent launch: at entry it lets the next
// kernel on the stream start, and before waiting for its own predecessor it
// only prefetches its weights into L2 (a non-binding prefetch, correct whatever
// the predecessor writes), so consecutive layers stream weights while the
// previous one finishes.  After the wait it quantises the activations itself
// (per-token absmax over x, then int8 into shared memory, interleaved in
// 16-element blocks in the order of expand_codes() and stored word-major: the
// 16-byte unit of block 4c + w at position w * CPR + c, so the lanes of a row
// read consecutive units).
//
// Arithmetic per 32-bit weight word (16 weights).  Up to three tokens: for
// j = 0..3 the masks w & (0x01010101 << 2j) and w & (0x02020202 << 2j) pick
// the +1 and -1 codes of weights 4b + j (scaled by 4^j and 2 * 4^j); one
// unsigned-by-signed dp4a each against interleaved activation word j
// accumulates them, and the scales are removed exactly (every partial is a
// multiple of its power of two) before the L-lane shuffle reduction.  Four
// tokens or more: the word is expanded once into four int8x4 words of
// {-1, 0, +1} and each token takes four signed dp4a, which costs less once
// the expansion is shared by enough tokens.
#include "sbl_common.cuh"

namespace sbl {

constexpr int kDecodeThreads = 512;
constexpr int kDecodeWarps = kDecodeThreads / 32;
constexpr int kDecodeBatch = 4;      // chunks per lane in flight
constexpr int kDecodeBatchWide = 16; // the same for calls too large for one batch per lane (one block per SM)
constexpr int kDecodeMaxGroup = 8;  // weight matrices per launch
// Two blocks of one-token passes share an SM, so the next call's blocks can
// start (and prefetch their weights) while this one drains.
// Blocks of kDecodeThreads threads; the wide batches use blocks of 128 (about
// 128 registers a thread, four blocks per SM), so a large call spreads its
// warps over every SM.
template <int NB>
constexpr int decode_threads() { return NB > kDecodeBatch ? 128 : kDecodeThreads; }
template <int TT, int NB>
constexpr int decode_min_blocks() { return NB > kDecodeBatch ? 4 : (TT == 1 ? 2 : 1); }

template <int CW>
__device__ __forceinline__ void load_chunk_words(const uint8_t* prow, int c, uint32_t (&w)[CW]) {
    if constexpr (CW == 4) {
        const uint4 v = ldg_stream(prow + 16 * c);
        w[0] = v.x;
        w[1 % CW] = v.y;
        w[2 % CW] = v.z;
        w[3 % CW] = v.w;
    } else {
        w[0] = __ldg(reinterpret_cast<const unsigned int*>(prow) + c);
    }
}

// The weight matrices of one launch: G matrices that share the activations x,
// their rows stacked (matrix g owns the rows row_end[g - 1] .. row_end[g] - 1
// of the launch), each with its own codes, scales and outputs.  A single
// layer is G = 1.
struct DecodeGroup {
    const uint8_t* packed[kDecodeMaxGroup];
    const float* row_scale[kDecodeMaxGroup];
    void* y[kDecodeMaxGroup];
    int32_t* acc_out[kDecodeMaxGroup];
    long long O[kDecodeMaxGroup];
    long long row_end[kDecodeMaxGroup];
    int G;
};

template <int L, int TT, int CW, int NB>
__global__ void __launch_bounds__(decode_threads<NB>(), decode_min_blocks<TT, NB>()) decode_kernel(const DecodeGroup grp, int K,
                                                                const uint16_t* __restrict__ x, long long T,
                                                                long long t0, int y_bf16, unsigned* status) {
    extern __shared__ uint4 xs[];  // TT x K/16 units of quantised activations (decode layout)
    constexpr int NTH = decode_threads<NB>();
    constexpr int NWP = NTH / 32;
    __shared__ uint32_t red[NWP][TT];
    __shared__ float s_sh[TT];
    asm volatile("griddepcontrol.launch_dependents;");
    constexpr int RW = 32 / L;
    const int CPR = K / (16 * CW);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / L, li = lane % L;
    const long long gr = static_cast<long long>(blockIdx.x) * NWP + warp;
    const long long grow = gr * RW + sub;  // row of the stacked matrices
    const bool valid = grow < grp.row_end[grp.G - 1];
    // the matrix this row belongs to (constant indices only: no local copy of the group)
    const uint8_t* packed = grp.packed[0];
    const float* row_scale = grp.row_scale[0];
    void* y = grp.y[0];
    int32_t* acc_out = grp.acc_out[0];
    long long O = grp.O[0], row = grow;
    if (grp.G > 1)
#pragma unroll
    for (int i = 1; i < kDecodeMaxGroup; ++i)
        if (i < grp.G && grow >= grp.row_end[i - 1]) {
            packed = grp.packed[i];
            row_scale = grp.row_scale[i];
            y = grp.y[i];
            acc_out = grp.acc_out[i];
            O = grp.O[i];
            row = grow - grp.row_end[i - 1];
        }
    const uint8_t* prow = packed + (valid ? row : 0) * (K >> 2);

    // Before the dependency wait: warm L2 with this lane's first batch of weights.
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int c = li + b * L;
        if (valid && c < CPR) asm volatile("prefetch.global.L2 [%0];" ::"l"(prow + 4 * CW * c));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    uint32_t wb[NB][CW];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int c = li + b * L;
        if (valid && c < CPR) load_chunk_words<CW>(prow, c, wb[b]);
        else
#pragma unroll
            for (int w = 0; w < CW; ++w) wb[b][w] = 0u;
    }
    // the row scale is needed only by the epilogue: load it now, off the critical path
    const float sc = (valid && li == 0) ? row_scale[row] : 0.0f;

    // Quantise this pass's tokens: per-token absmax, then int8 into shared memory.
    const int nvec = K >> 3;
    const int nblk = K >> 4;
    if (TT == 1 && nblk <= NTH) {
        // one token, K <= 8192: each thread keeps its 16-element block in
        // registers between the absmax and the quantisation
        constexpr int XB = 1;
        const long long tt = t0 < T ? t0 : T - 1;
        const uint4* xr = reinterpret_cast<const uint4*>(x + tt * K);
        uint4 xa[XB][2];
        uint32_t mx = 0;
#pragma unroll
        for (int i = 0; i < XB; ++i) {
            const int b = threadIdx.x + i * NTH;
            if (b < nblk) {
                xa[i][0] = ldg_nc(xr + 2 * b);
                xa[i][1] = ldg_nc(xr + 2 * b + 1);
                mx = absmax8(xa[i][1], absmax8(xa[i][0], mx));
            }
        }
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0) red[warp][0] = mx;
        __syncthreads();
        mx = 0;
#pragma unroll
        for (int w = 0; w < NWP; ++w) mx = max(mx, red[w][0]);
        const float st = __fdiv_rn(127.0f, fmaxf(__uint_as_float(mx << 16), 1e-5f));
        if (threadIdx.x == 0) {
            if (mx >= 0x7F80u && blockIdx.x == 0) raise_status(status, kStatusNonfinite);
            s_sh[0] = st;
        }
#pragma unroll
        for (int i = 0; i < XB; ++i) {
            const int b = threadIdx.x + i * NTH;
            if (b < nblk) {
                const int pos = CW == 4 ? (b & 3) * CPR + (b >> 2) : b;
                xs[pos] = quant_block16<true>(xa[i][0], xa[i][1], st);
            }
        }
        __syncthreads();
    } else {
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            const long long tt = t0 + t < T ? t0 + t : T - 1;
            const uint4* xr = reinterpret_cast<const uint4*>(x + tt * K);
            uint32_t mx = 0;
            for (int v = threadIdx.x; v < nvec; v += NTH) mx = absmax8(ldg_nc(xr + v), mx);
            mx = __reduce_max_sync(0xFFFFFFFFu, mx);
            if (lane == 0) red[warp][t] = mx;
        }
        __syncthreads();
        if (threadIdx.x < TT) {
            uint32_t mx = 0;
#pragma unroll
            for (int w = 0; w < NWP; ++w) mx = max(mx, red[w][threadIdx.x]);
            if (mx >= 0x7F80u && blockIdx.x == 0) raise_status(status, kStatusNonfinite);
            s_sh[threadIdx.x] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(mx << 16), 1e-5f));
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            const long long tt = t0 + t < T ? t0 + t : T - 1;
            const uint4* xr = reinterpret_cast<const uint4*>(x + tt * K);
            const float st = s_sh[t];
            for (int b = threadIdx.x; b < nblk; b += NTH) {
                const int pos = CW == 4 ? (b & 3) * CPR + (b >> 2) : b;
                xs[t * nblk + pos] = quant_block16<true>(ldg_nc(xr + 2 * b), ldg_nc(xr + 2 * b + 1), st);
            }
        }
        __syncthreads();
    }

    // Four or more tokens: expand each code word once into int8 {-1, 0, +1}
    // (expand_codes, word j = weights 4b + j) and take one signed dp4a per
    // activation word and token.  Fewer tokens: split the +1 and -1 codes with
    // masks (no expansion) and remove their power-of-two scales afterwards.
    constexpr bool EXPAND = TT >= 4;
    int acc[TT];
    int alo[EXPAND ? 1 : TT][4], ahi[EXPAND ? 1 : TT][4];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0;
#pragma unroll
    for (int t = 0; t < (EXPAND ? 1 : TT); ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) alo[t][j] = ahi[t][j] = 0;

    for (int c0 = li; c0 < CPR; c0 += NB * L) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int c = c0 + b * L;
            if (c >= CPR) break;
#pragma unroll
            for (int w = 0; w < CW; ++w) {
                const uint32_t word = wb[b][w];
                if constexpr (EXPAND) {
                    uint32_t e[4];
                    expand_codes(word, e);
#pragma unroll
                    for (int t = 0; t < TT; ++t) {
                        const uint4 xv = xs[t * nblk + w * CPR + c];
                        acc[t] = __dp4a(static_cast<int>(e[0]), static_cast<int>(xv.x), acc[t]);
                        acc[t] = __dp4a(static_cast<int>(e[1]), static_cast<int>(xv.y), acc[t]);
                        acc[t] = __dp4a(static_cast<int>(e[2]), static_cast<int>(xv.z), acc[t]);
                        acc[t] = __dp4a(static_cast<int>(e[3]), static_cast<int>(xv.w), acc[t]);
                    }
                } else {
                    uint32_t mlo[4], mhi[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        mlo[j] = word & (0x01010101u << (2 * j));
                        mhi[j] = word & (0x02020202u << (2 * j));
                    }
#pragma unroll
                    for (int t = 0; t < TT; ++t) {
                        const uint4 xv = xs[t * nblk + w * CPR + c];
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            alo[EXPAND ? 0 : t][j] = dp4a_us(mlo[j], xw[j], alo[EXPAND ? 0 : t][j]);
                            ahi[EXPAND ? 0 : t][j] = dp4a_us(mhi[j], xw[j], ahi[EXPAND ? 0 : t][j]);
                        }
                    }
                }
            }
        }
        const int cn = c0 + NB * L;
        if (cn < CPR) {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int c = cn + b * L;
                if (valid && c < CPR) load_chunk_words<CW>(prow, c, wb[b]);
                else
#pragma unroll
                    for (int w = 0; w < CW; ++w) wb[b][w] = 0u;
            }
        }
    }

#pragma unroll
    for (int t = 0; t < TT; ++t) {
        int a = acc[t];
        if constexpr (!EXPAND) {
#pragma unroll
            for (int j = 0; j < 4; ++j) a += (alo[t][j] >> (2 * j)) - (ahi[t][j] >> (2 * j + 1));
        }
#pragma unroll
        for (int off = L / 2; off >= 1; off >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, off);
        acc[t] = a;
    }
    if (valid && li == 0) {
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            const long long tt = t0 + t;
            if (tt < T) {
                const float v = __fdiv_rn(__fmul_rn(static_cast<float>(acc[t]), sc), s_sh[t]);
                if (y_bf16)
                    reinterpret_cast<__nv_bfloat16_raw*>(y)[tt * O + row] =
                        static_cast<__nv_bfloat16_raw>(__float2bfloat16_rn(v));
                else
                    reinterpret_cast<float*>(y)[tt * O + row] = v;
                if (acc_out) acc_out[tt * O + row] = acc[t];
            }
        }
    }
}

// Lanes per row and chunks per lane in flight.  A call should fit in one block
// of kDecodeWarps warps per SM, which leaves room on each SM for the next
// call's block, with every load in flight at once: among the lane counts whose
// warps fit, take the best chunk utilisation per batch of loads (ties: more
// lanes per row).  A call too large for that (several batches per lane: big
// layers, or several layers in one grouped launch) of one or two tokens takes
// batches of kDecodeBatchWide chunks (more registers: 16 warps per SM in
// blocks of four) when that needs fewer batches.
struct DecodePlan {
    int L;
    int NB;
};

static DecodePlan choose_plan(long long O, int cpr, int num_sms, int tt, bool wide) {
    auto best_for = [&](int nb, long long cap, int& batches) {
        int best = 1;
        double best_score = -1.0;
        batches = 1 << 30;
        for (int L = 32; L >= 1; L >>= 1) {
            const long long warps = (O + (32 / L) - 1) / (32 / L);
            if (warps > cap) continue;
            const int per_lane = (cpr + L - 1) / L;
            const double eff = static_cast<double>(cpr) / (static_cast<double>(per_lane) * L);
            const int nbat = (per_lane + nb - 1) / nb;
            const double score = eff / nbat;
            if (score > best_score + 1e-9) {
                best_score = score;
                best = L;
                batches = nbat;
            }
        }
        return best;
    };
    const long long cap = static_cast<long long>(num_sms) * kDecodeWarps;
    int b1 = 0;
    const int L1 = best_for(kDecodeBatch, cap, b1);
    if (tt <= 2 && wide && b1 > 1) {
        int b2 = 0;
        const int L2 = best_for(kDecodeBatchWide, cap, b2);
        if (b2 < b1) return {L2, kDecodeBatchWide};
    }
    return {L1, kDecodeBatch};
}

template <int L, int TT, int CW, int NB>
static cudaError_t launch_decode_lt(const DecodeGroup& grp, int K, const uint16_t* x, long long T, long long t0,
                                    int y_bf16, unsigned* status, cudaStream_t stream) {
    constexpr int RW = 32 / L;
    const long long rows = grp.row_end[grp.G - 1];
    const long long groups = (rows + RW - 1) / RW;
    constexpr int NTH = decode_threads<NB>();
    const long long blocks = (groups + NTH / 32 - 1) / (NTH / 32);
    const size_t smem = static_cast<size_t>(TT) * K;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<L, TT, CW, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<L, TT, CW, NB>, grp, K, x, T, t0, y_bf16, status);
}

template <int TT, int CW, int NB>
static cudaError_t launch_decode_t(int L, const DecodeGroup& grp, int K, const uint16_t* x, long long T,
                                   long long t0, int y_bf16, unsigned* status, cudaStream_t stream) {
#define SBL_DECODE_CASE(LV) \
    case LV: return launch_decode_lt<LV, TT, CW, NB>(grp, K, x, T, t0, y_bf16, status, stream);
    switch (L) {
        SBL_DECODE_CASE(32)
        SBL_DECODE_CASE(16)
        SBL_DECODE_CASE(8)
        SBL_DECODE_CASE(4)
        SBL_DECODE_CASE(2)
        default: return launch_decode_lt<1, TT, CW, NB>(grp, K, x, T, t0, y_bf16, status, stream);
    }
#undef SBL_DECODE_CASE
}

template <int TT>
static cudaError_t launch_decode_cw(const DecodePlan& plan, bool wide, const DecodeGroup& grp, int K,
                                    const uint16_t* x, long long T, long long t0, int y_bf16, unsigned* status,
                                    cudaStream_t stream) {
    if (wide) {
        if constexpr (TT <= 2) {
            if (plan.NB == kDecodeBatchWide)
                return launch_decode_t<TT, 4, kDecodeBatchWide>(plan.L, grp, K, x, T, t0, y_bf16, status, stream);
        }
        return launch_decode_t<TT, 4, kDecodeBatch>(plan.L, grp, K, x, T, t0, y_bf16, status, stream);
    }
    return launch_decode_t<TT, 1, kDecodeBatch>(plan.L, grp, K, x, T, t0, y_bf16, status, stream);
}

// Decode of G weight matrices that share x, for any T: passes of up to 8
// tokens (later passes re-read the weights, mostly from L2).  Needs
// K % 16 == 0, TT * K bytes of shared memory and 1 <= G <= kDecodeMaxGroup.
static cudaError_t launch_decode_group(const DecodeGroup& grp, long long K, const uint16_t* x, long long T,
                                       int y_bf16, int num_sms, cudaStream_t stream, unsigned* status) {
    const int Ki = static_cast<int>(K);
    const bool wide = (Ki % 64) == 0;
    const int cpr = wide ? Ki / 64 : Ki / 16;
    const long long rows = grp.row_end[grp.G - 1];
    for (long long t0 = 0; t0 < T; t0 += 8) {
        const long long rem = T - t0;
        const int tt = rem > 4 ? 8 : rem > 2 ? 4 : static_cast<int>(rem);
        const DecodePlan plan = choose_plan(rows, cpr, num_sms, tt, wide);
        cudaError_t e;
        if (tt == 8) e = launch_decode_cw<8>(plan, wide, grp, Ki, x, T, t0, y_bf16, status, stream);
        else if (tt == 4) e = launch_decode_cw<4>(plan, wide, grp, Ki, x, T, t0, y_bf16, status, stream);
        else if (tt == 2) e = launch_decode_cw<2>(plan, wide, grp, Ki, x, T, t0, y_bf16, status, stream);
        else e = launch_decode_cw<1>(plan, wide, grp, Ki, x, T, t0, y_bf16, status, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_decode(const uint8_t* packed, const float* row_scale, long long O, long long K,
                          const uint16_t* x, long long T, void* y, int y_bf16, int32_t* acc_out, unsigned* status,
                          int num_sms, cudaStream_t stream) {
    DecodeGroup grp = {};
    grp.packed[0] = packed;
    grp.row_scale[0] = row_scale;
    grp.y[0] = y;
    grp.acc_out[0] = acc_out;
    grp.O[0] = O;
    grp.row_end[0] = O;
    grp.G = 1;
    return launch_decode_group(grp, K, x, T, y_bf16, num_sms, stream, status);
}

int decode_max_group() { return kDecodeMaxGroup; }

// G matrices (G <= decode_max_group()) that share x, in one launch per pass of
// up to 8 tokens; matrix g has O[g] rows and its own packed, row_scale, y and
// acc_out (which may be null).
cudaError_t launch_decode_grouped(int G, const uint8_t* const* packed, const float* const* row_scale,
                                  const long long* O, long long K, const uint16_t* x, long long T, void* const* y,
                                  int y_bf16, int32_t* const* acc_out, unsigned* status, int num_sms,
                                  cudaStream_t stream) {
    if (G < 1 || G > kDecodeMaxGroup) return cudaErrorInvalidValue;
    DecodeGroup grp = {};
    long long end = 0;
    for (int g = 0; g < G; ++g) {
        grp.packed[g] = packed[g];
        grp.row_scale[g] = row_scale[g];
        grp.y[g] = y[g];
        grp.acc_out[g] = acc_out ? acc_out[g] : nullptr;
        grp.O[g] = O[g];
        end += O[g];
        grp.row_end[g] = end;
    }
    grp.G = G;
    if (end == 0) return cudaSuccess;
    return launch_decode_group(grp, K, x, T, y_bf16, num_sms, stream, status);
}

}  // namespace sbl
