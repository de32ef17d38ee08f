// Decode path for a few tokens (T <= 16 per pass) on the warp-level int8 MMA.
//
// Same result as the CUDA-core decode kernel (decode.cu): the integer product
// of the Sparse-BitNet Guide's linear-evaluation equation ("Mathematical
// Formulation of Sparse-BitLinear") over 2-bit weights read once from HBM,
// with the activations quantised per token inside the kernel (or, after the
// RMSNorm front end, copied in already quantised) and the dequant epilogue
// fused.  With several tokens the CUDA-core form spends four dp4a per
// 16 weights and token plus a shared-memory load per token; here the ternary
// codes are expanded once into int8 registers that are the A fragments of
// mma.sync m16n8k32 (16 output rows x 32 weights), and the activations of up
// to 8 tokens are one B fragment, so the per-token arithmetic leaves the
// integer pipes.
//
// Work split: a warp owns a tile of 16 output rows and a slice of its chunks
// (a chunk = 64 * CW weights of each row: thread (g, t) of the warp holds CW
// consecutive 32-bit code words of rows g and g + 8).  KS warps of one block
// share a row tile and their int32 partial tiles are summed in shared memory.
//
// Expansion: code word w (weights 0..15 of a 16-weight block) becomes four
// int8x4 words with expand_pairs() (one byte permute each: weights 0,2,4,6;
// 1,3,5,7; 8,10,12,14; 9,11,13,15).  The MMA sums over k in any order as long
// as the A and B fragments of one thread agree, so the activations of each
// 16-element block are stored in that same order (quant_block16_pairs).  In shared memory token n's blocks sit at
// n * S, S = K bytes padded to 64 mod 128 so that the two tokens of a
// quarter-warp read disjoint banks, and within a chunk the block of thread t's
// i-th word sits at 4 i + t, so the four threads of a group read 64
// contiguous bytes.
//
// The kernel is a programmatic dependent launch, like the CUDA-core decode: it
// lets the next kernel start at entry and prefetches all of its weights into
// L2 (non-binding) before waiting for its predecessor.
#include "sbl_common.cuh"

namespace sbl {

constexpr int kDmThreads = 512;
constexpr int kDmWarps = kDmThreads / 32;
constexpr int kDmBatch = 4;                       // chunks of one warp loaded together
constexpr int kDmMinBlocks = 1;                   // blocks per SM the register budget allows
constexpr int kDmMaxTokens = 16;                  // tokens of one pass (two n8 tiles)

// Shared-memory stride of one token's activations (K % 64 == 0).
__host__ __device__ inline int dm_stride(int K) { return (K % 128 == 64) ? K : K + 64; }

__host__ __device__ inline size_t dm_smem_bytes(int K, int TP, int NT) {
    return static_cast<size_t>(TP) * dm_stride(K) + static_cast<size_t>(kDmWarps) * 32 * 4 * NT * 4;
}

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int CW>
__device__ __forceinline__ void load_words(const uint8_t* p, bool ok, uint32_t (&w)[CW]) {
    if (!ok) {
#pragma unroll
        for (int i = 0; i < CW; ++i) w[i] = 0u;
        return;
    }
    if constexpr (CW == 4) {
        const uint4 v = ldg_stream(p);
        w[0] = v.x;
        w[1 % CW] = v.y;
        w[2 % CW] = v.z;
        w[3 % CW] = v.w;
    } else if constexpr (CW == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = v.x;
        w[1 % CW] = v.y;
    } else {
        w[0] = __ldg(reinterpret_cast<const unsigned int*>(p));
    }
}

// PREQ: the activations arrive already quantised (x_q int8 [T, K] with each
// 16-element block in the pairing order, and s_tok [T], from the RMSNorm
// front end) and are only copied into shared memory.
template <int NT, int CW, bool PREQ>
__global__ void __launch_bounds__(kDmThreads, kDmMinBlocks)
    decode_mma_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ row_scale, int O, int K,
                      const uint16_t* __restrict__ x, const int8_t* __restrict__ xq_in,
                      const float* __restrict__ stok_in, int t0, int TP, int KS, void* __restrict__ y, int y_bf16,
                      int32_t* __restrict__ acc_out, unsigned* status) {
    extern __shared__ __align__(16) uint8_t dm_smem[];
    __shared__ uint32_t red_max[kDmWarps];
    __shared__ float s_sh[kDmMaxTokens];
    asm volatile("griddepcontrol.launch_dependents;");
    const int S = dm_stride(K);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, tg = lane & 3;
    const int C = K / (64 * CW);
    const int ks = warp % KS;
    const int rt = blockIdx.x * (kDmWarps / KS) + warp / KS;
    const int r0 = rt * 16 + g, r1 = r0 + 8;
    const bool v0 = r0 < O, v1 = r1 < O;
    const size_t rowb = static_cast<size_t>(K) >> 2;
    const uint8_t* p0 = packed + static_cast<size_t>(v0 ? r0 : 0) * rowb + tg * 4 * CW;
    const uint8_t* p1 = packed + static_cast<size_t>(v1 ? r1 : 0) * rowb + tg * 4 * CW;
    const int nck = ks < C ? (C - ks + KS - 1) / KS : 0;

    // Before the dependency wait: pull this warp's weights into L2.
    for (int j = 0; j < nck; ++j) {
        const int c = ks + j * KS;
        if (v0) asm volatile("prefetch.global.L2 [%0];" ::"l"(p0 + c * 16 * CW));
        if (v1) asm volatile("prefetch.global.L2 [%0];" ::"l"(p1 + c * 16 * CW));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    constexpr int NB = CW == 4 ? 2 : kDmBatch;  // chunks loaded together (8 or 16 code words per thread)
    uint32_t wa[NB][CW], wb[NB][CW];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int c = ks + b * KS;
        load_words<CW>(p0 + c * 16 * CW, v0 && b < nck, wa[b]);
        load_words<CW>(p1 + c * 16 * CW, v1 && b < nck, wb[b]);
    }
    // the row scales are needed only by the epilogue: load them now
    const float sc0 = (v0 && ks == 0) ? row_scale[r0] : 0.0f;
    const float sc1 = (v1 && ks == 0) ? row_scale[r1] : 0.0f;

    const int nblk = K >> 4;
    auto pos = [](int blk) {  // shared-memory slot of 16-element block blk of a token
        const int c = blk / (4 * CW), l = blk % (4 * CW);
        return c * 4 * CW + (l % CW) * 4 + l / CW;
    };
    if constexpr (PREQ) {
        for (int u = threadIdx.x; u < TP * nblk; u += kDmThreads) {
            const int tok = u / nblk, blk = u - tok * nblk;
            reinterpret_cast<uint4*>(dm_smem + static_cast<size_t>(tok) * S)[pos(blk)] =
                __ldg(reinterpret_cast<const uint4*>(xq_in + static_cast<size_t>(t0 + tok) * K) + blk);
        }
        if (threadIdx.x < TP) s_sh[threadIdx.x] = stok_in[t0 + threadIdx.x];
        __syncthreads();
    } else {
        // Quantise the pass's TP tokens: 16 / TP warps per token, each thread
        // keeping up to four 16-element blocks in registers between the absmax and
        // the quantisation (blocks beyond that are read again, four at a time).
        const int wpt = kDmWarps / TP;
        const int qt = warp / wpt;
        const bool qw = qt < TP;
        const int qj = (warp - qt * wpt) * 32 + lane;
        const int nthr = wpt * 32;
        const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + (qw ? qt : 0)) * K);
        constexpr int XB = 4;
        uint4 xa[XB][2];
        uint32_t mx = 0;
        if (qw) {
    #pragma unroll
            for (int i = 0; i < XB; ++i) {
                const int b = qj + i * nthr;
                if (b < nblk) {
                    xa[i][0] = ldg_nc(xr + 2 * b);
                    xa[i][1] = ldg_nc(xr + 2 * b + 1);
                    mx = absmax8(xa[i][1], absmax8(xa[i][0], mx));
                }
            }
    #pragma unroll 4
            for (int b = qj + XB * nthr; b < nblk; b += nthr) mx = absmax8(ldg_nc(xr + 2 * b + 1), absmax8(ldg_nc(xr + 2 * b), mx));
        }
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0) red_max[warp] = mx;
        __syncthreads();
        if (threadIdx.x < TP) {
            uint32_t m = 0;
    #pragma unroll
            for (int w = 0; w < kDmWarps; ++w)
                if (w / wpt == static_cast<int>(threadIdx.x)) m = max(m, red_max[w]);
            if (m >= 0x7F80u && blockIdx.x == 0) raise_status(status, kStatusNonfinite);
            s_sh[threadIdx.x] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(m << 16), 1e-5f));
        }
        __syncthreads();
        if (qw) {
            const float st = s_sh[qt];
            uint4* xt = reinterpret_cast<uint4*>(dm_smem + static_cast<size_t>(qt) * S);
    #pragma unroll
            for (int i = 0; i < XB; ++i) {
                const int b = qj + i * nthr;
                if (b < nblk) xt[pos(b)] = quant_block16_pairs(xa[i][0], xa[i][1], st);
            }
    #pragma unroll 4
            for (int b = qj + XB * nthr; b < nblk; b += nthr)
                xt[pos(b)] = quant_block16_pairs(ldg_nc(xr + 2 * b), ldg_nc(xr + 2 * b + 1), st);
        }
        __syncthreads();
    }

    int acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[nt][r] = 0;

    for (int j0 = 0; j0 < nck; j0 += NB) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            if (j0 + b >= nck) break;
            const int c = ks + (j0 + b) * KS;
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                uint32_t ea[4], eb[4];
                expand_pairs(wa[b][i], ea);
                expand_pairs(wb[b][i], eb);
                const int unit = c * 4 * CW + i * 4 + tg;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int tok = nt * 8 + g;
                    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
                    if (tok < TP) xv = reinterpret_cast<const uint4*>(dm_smem + static_cast<size_t>(tok) * S)[unit];
                    mma_s8_16832(acc[nt], ea[0], eb[0], ea[1], eb[1], xv.x, xv.y);
                    mma_s8_16832(acc[nt], ea[2], eb[2], ea[3], eb[3], xv.z, xv.w);
                }
            }
        }
        if (j0 + NB < nck) {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int j = j0 + NB + b;
                const int c = ks + j * KS;
                load_words<CW>(p0 + c * 16 * CW, v0 && j < nck, wa[b]);
                load_words<CW>(p1 + c * 16 * CW, v1 && j < nck, wb[b]);
            }
        }
    }

    // Sum the KS partial tiles of a row tile (warps ks = 1.. hand theirs to ks = 0).
    if (KS > 1) {
        int* red = reinterpret_cast<int*>(dm_smem + static_cast<size_t>(TP) * S);
        if (ks != 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) red[(warp * 4 * NT + nt * 4 + r) * 32 + lane] = acc[nt][r];
        }
        __syncthreads();
        if (ks == 0) {
            for (int k2 = 1; k2 < KS; ++k2)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) acc[nt][r] += red[((warp + k2) * 4 * NT + nt * 4 + r) * 32 + lane];
        }
    }
    if (ks != 0) return;

    // Dequantise: y[t, o] = acc * row_scale[o] / s_tok[t].  Thread (g, t) holds
    // rows g, g + 8 and tokens 2t, 2t + 1 of each n8 tile.
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int tok = nt * 8 + 2 * tg + h;
            if (tok >= TP) continue;
            const size_t tt = static_cast<size_t>(t0 + tok);
            const float st = s_sh[tok];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const bool ok = half ? v1 : v0;
                if (!ok) continue;
                const int row = half ? r1 : r0;
                const int a = acc[nt][2 * half + h];
                const float v = __fdiv_rn(__fmul_rn(static_cast<float>(a), half ? sc1 : sc0), st);
                if (y_bf16)
                    reinterpret_cast<__nv_bfloat16_raw*>(y)[tt * O + row] =
                        static_cast<__nv_bfloat16_raw>(__float2bfloat16_rn(v));
                else
                    reinterpret_cast<float*>(y)[tt * O + row] = v;
                if (acc_out) acc_out[tt * O + row] = a;
            }
        }
    }
}

// Warps per row tile: the fewest whose chunk slices fit one load batch, then
// more while the grid still has fewer blocks than SMs (more SMs stream the
// weights), never more warps than chunks.
static int choose_ks(int R, int C, int nb, int num_sms) {
    int ks = 1;
    while (ks < kDmWarps && ks < C && (C + ks - 1) / ks > nb) ks *= 2;
    while (ks < kDmWarps && 2 * ks <= C) {
        const long long blocks = (static_cast<long long>(R) * 2 * ks + kDmWarps - 1) / kDmWarps;
        if (blocks > num_sms) break;
        ks *= 2;
    }
    return ks;
}

template <int NT, int CW, bool PREQ>
static cudaError_t launch_dm(const uint8_t* packed, const float* row_scale, int O, int K, const uint16_t* x,
                             const int8_t* xq_in, const float* stok_in, int t0,
                             int TP, int KS, void* y, int y_bf16, int32_t* acc_out, unsigned* status,
                             cudaStream_t stream) {
    const int R = (O + 15) / 16;
    const int tiles_per_block = kDmWarps / KS;
    const int blocks = (R + tiles_per_block - 1) / tiles_per_block;
    const size_t smem = dm_smem_bytes(K, TP, NT);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<NT, CW, PREQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(kDmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_mma_kernel<NT, CW, PREQ>, packed, row_scale, O, K, x, xq_in, stok_in, t0, TP, KS, y, y_bf16,
                              acc_out, status);
}

template <int NT, bool PREQ>
static cudaError_t launch_dm_cw(int CW, const uint8_t* packed, const float* row_scale, int O, int K,
                                const uint16_t* x, const int8_t* xq_in, const float* stok_in, int t0, int TP, int KS,
                                void* y, int y_bf16, int32_t* acc_out, unsigned* status, cudaStream_t stream) {
    if (CW == 4)
        return launch_dm<NT, 4, PREQ>(packed, row_scale, O, K, x, xq_in, stok_in, t0, TP, KS, y, y_bf16, acc_out,
                                      status, stream);
    if (CW == 2)
        return launch_dm<NT, 2, PREQ>(packed, row_scale, O, K, x, xq_in, stok_in, t0, TP, KS, y, y_bf16, acc_out,
                                      status, stream);
    return launch_dm<NT, 1, PREQ>(packed, row_scale, O, K, x, xq_in, stok_in, t0, TP, KS, y, y_bf16, acc_out, status,
                                  stream);
}

bool decode_mma_supported(long long K) { return K % 64 == 0 && K > 0 && dm_smem_bytes(static_cast<int>(K), 1, 2) <= 200 * 1024; }

// Passes of up to 16 tokens (as many as fit 200 KB of shared memory); later
// passes read the weights again, mostly from L2.  Needs K % 64 == 0.  With
// xq_in (and stok_in) the activations come already quantised (pairing order)
// and x is not read.
cudaError_t launch_decode_mma(const uint8_t* packed, const float* row_scale, long long O, long long K,
                              const uint16_t* x, long long T, void* y, int y_bf16, int32_t* acc_out, unsigned* status,
                              int num_sms, cudaStream_t stream, const int8_t* xq_in, const float* stok_in) {
    const int Ki = static_cast<int>(K), Oi = static_cast<int>(O);
    const int CW = (Ki % 256 == 0) ? 4 : (Ki % 128 == 0) ? 2 : 1;
    const int C = Ki / (64 * CW);
    const int R = (Oi + 15) / 16;
    const int KS = choose_ks(R, C, CW == 4 ? 2 : kDmBatch, num_sms);
    int cap = kDmMaxTokens;
    while (cap > 1 && dm_smem_bytes(Ki, cap, cap > 8 ? 2 : 1) > 200 * 1024) --cap;
    for (long long t0 = 0; t0 < T; t0 += cap) {
        const int TP = static_cast<int>(T - t0 < cap ? T - t0 : cap);
        const int t0i = static_cast<int>(t0);
        cudaError_t e;
        if (xq_in)
            e = TP > 8 ? launch_dm_cw<2, true>(CW, packed, row_scale, Oi, Ki, x, xq_in, stok_in, t0i, TP, KS, y, y_bf16,
                                               acc_out, status, stream)
                       : launch_dm_cw<1, true>(CW, packed, row_scale, Oi, Ki, x, xq_in, stok_in, t0i, TP, KS, y, y_bf16,
                                               acc_out, status, stream);
        else
            e = TP > 8 ? launch_dm_cw<2, false>(CW, packed, row_scale, Oi, Ki, x, nullptr, nullptr, t0i, TP, KS, y,
                                                y_bf16, acc_out, status, stream)
                       : launch_dm_cw<1, false>(CW, packed, row_scale, Oi, Ki, x, nullptr, nullptr, t0i, TP, KS, y,
                                                y_bf16, acc_out, status, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace sbl
