// Prefill path for 2:4 weights on the structured-sparse tensor cores:
// acc[t, o] = sum_k W_t[o, k] * x_q[t, k] with tcgen05.mma.sp (kind::i8), then
// y = acc * scale_o / s_t.
//
// The Sparse-BitNet Guide, "The Hardware Mechanics of 2:4 Sparsity": with at
// most two nonzeros in every four consecutive weights, the tensor cores take
// the two kept values of each group plus a 4-bit index word and do half the
// multiply-adds of the dense product.  The sparse operand of the instruction
// is A, so here the weights are A (M = 128 output rows per CTA) and the
// activations B (N = 192 tokens); the accumulator rows in tensor memory are
// outputs, and the epilogue writes y transposed.
//
// 1. sp_compress_kernel turns the 2-bit codes of each group of four into two
//    int8 values and a nibble idx0 | idx1 << 2 (the kept positions, idx0 <
//    idx1; a group with one nonzero at position i keeps (i, 3), or (0, 3) when
//    i = 3; an all-zero group keeps (0, 0)), all in the call's workspace:
//    values int8 [O, K/2], nibbles [O, E_pitch] with E_pitch = 32 bytes per
//    256-deep k-block (zero padded).  Packed codes that hold three or more
//    nonzeros in a group are not 2:4 weights; the kernel reports
//    kStatusInvalid and zeroes such a group.
// 2. prefill_sp_kernel, persistent and warp-specialised, one CTA per SM:
//      warps 0-7  epilogue: warp w owns TMEM lanes 32(w % 4) .. + 31 (32 output
//                 rows) and every other 32-token slice (starting at w / 4);
//                 per slice tcgen05.ld (the next one in flight), dequantise
//                 into the warp's 32-token x 32-output box in shared memory
//                 (row = token) and write it with one TMA store
//      warps 8-11 metadata: each thread loads its row's 32 nibble bytes of the
//                 k-block and writes them into its TMEM lane with tcgen05.st
//      warp 12    TMA producer: compressed weight tile (128 rows x 128 bytes =
//                 256 k, SW128) and two activation tiles (192 tokens x 128 k,
//                 SW128)
//      warp 13    TMEM allocation and single-thread MMA issue: four
//                 M = 128, N = 192, K = 64 sparse MMAs per k-block
//    Tensor memory: two 192-column accumulators and 8 metadata columns per
//    stage (lane m, column c holds the nibbles of k 32c .. 32c + 31 of row m).
//
// Every wait is bounded; a CTA that gives up records a timeout and winds down.
#include <cuda.h>

#include <type_traits>

#include "sbl_common.cuh"
#include "tc_util.cuh"

namespace sbl {

namespace sp {
constexpr int BM = 128;                 // output rows per tile (MMA M, TMEM lanes)
constexpr int BN = 192;                 // tokens per tile (MMA N)
constexpr int BK = 256;                 // logical k per stage
constexpr int A_BYTES = BM * BK / 2;    // compressed weights: 128 rows x 128 bytes
constexpr int B_HALF = BN * 128;        // one 128-deep activation sub-tile
constexpr int B_BYTES = 2 * B_HALF;
constexpr int E_BYTES_ROW = BK / 8;     // nibble bytes per row per stage
constexpr int STAGES = 3;
constexpr int EPI_WARPS = 8;            // two per TMEM lane quadrant
constexpr int META_WARPS = 4;
constexpr int WARP_META = EPI_WARPS;
constexpr int WARP_TMA = WARP_META + META_WARPS;
constexpr int WARP_MMA = WARP_TMA + 1;
constexpr int THREADS = (WARP_MMA + 1) * 32;
constexpr int E_COL0 = 2 * BN;          // metadata columns after the accumulators
constexpr int TMEM_COLS = 512;
static_assert(E_COL0 + STAGES * (BK / 32) <= TMEM_COLS, "tensor memory columns");
}  // namespace sp

// Bytes of compressed values and of nibbles per row, as laid out in the workspace.
__host__ __device__ inline long long sp_values_pitch(long long K) { return K / 2; }
__host__ __device__ inline long long sp_meta_pitch(long long K) { return (K + sp::BK - 1) / sp::BK * sp::E_BYTES_ROW; }

// ---------------------------------------------------------------------------
// compression: one thread per 32-bit word of codes (16 weights, four groups)
__global__ void sp_compress_kernel(const uint32_t* __restrict__ packed, long long O, long long K,
                                   uint16_t* __restrict__ values, uint8_t* __restrict__ meta, unsigned* status) {
    const long long words_per_row = K / 16;
    const long long e_pitch = sp_meta_pitch(K);
    const long long total = O * (e_pitch / 2);  // one thread per 16 k of the padded nibble row
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long row = i / (e_pitch / 2);
        const long long w = i % (e_pitch / 2);
        uint32_t nib = 0;
        if (w < words_per_row) {
            const uint32_t codes = packed[row * words_per_row + w];
            uint32_t vals[4];
            bool bad = false;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const uint32_t c = (codes >> (8 * g)) & 0xFFu;
                int idx[2] = {0, 0};
                int v[2] = {0, 0};
                int cnt = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t q = (c >> (2 * j)) & 3u;
                    if (q != 0u) {
                        if (cnt < 2) {
                            idx[cnt] = j;
                            v[cnt] = q == 1u ? 1 : -1;
                        }
                        ++cnt;
                    }
                }
                if (cnt > 2) {
                    bad = true;
                    idx[0] = idx[1] = 0;
                    v[0] = v[1] = 0;
                } else if (cnt == 1) {
                    if (idx[0] == 3) {
                        idx[1] = 3;
                        v[1] = v[0];
                        idx[0] = 0;
                        v[0] = 0;
                    } else {
                        idx[1] = 3;
                    }
                }
                vals[g] = (static_cast<uint32_t>(v[0]) & 0xFFu) | ((static_cast<uint32_t>(v[1]) & 0xFFu) << 8);
                nib |= static_cast<uint32_t>(idx[0] | (idx[1] << 2)) << (4 * g);
            }
            if (bad) raise_status(status, kStatusInvalid);
            uint2 out;
            out.x = vals[0] | (vals[1] << 16);
            out.y = vals[2] | (vals[3] << 16);
            *reinterpret_cast<uint2*>(values + (row * (K / 2) + 8 * w) / 2) = out;
        }
        *reinterpret_cast<uint16_t*>(meta + row * e_pitch + 2 * w) = static_cast<uint16_t>(nib);
    }
}

// ---------------------------------------------------------------------------
// sparse GEMM
struct SpSmem {
    uint8_t a[sp::STAGES][sp::A_BYTES];     // 1024-byte aligned tiles
    uint8_t b[sp::STAGES][sp::B_BYTES];
    uint8_t ybox[sp::EPI_WARPS][32 * 128];  // per-warp output box: 32 tokens x 32 outputs
    uint64_t full_tma[sp::STAGES];
    uint64_t full_meta[sp::STAGES];
    uint64_t empty[sp::STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t sp_smem_bytes() { return sizeof(SpSmem) + 1024; }
static_assert(sp_smem_bytes() <= 232448, "sparse prefill tile does not fit in shared memory");

// Sparse instruction descriptor: s8 x s8 -> s32, K-major, M = 128, N = BN,
// sparse flag (bit 2), metadata selector 0.
__device__ __forceinline__ uint32_t sp_idesc() {
    return (1u << 2) | (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(sp::BN >> 3) << 17) |
           (static_cast<uint32_t>(sp::BM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_sp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                          uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%5], %3, {%6, %6, %6, %6}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(e_tmem), "r"(0u)
        : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__global__ void __launch_bounds__(sp::THREADS, 1)
    prefill_sp_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_y, int y_vec, const uint8_t* __restrict__ meta, long long e_pitch, const float* __restrict__ row_scale,
                      const float* __restrict__ s_tok, int T, int O, int K, void* __restrict__ y, int y_bf16,
                      int32_t* __restrict__ acc_out, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    auto* sm = reinterpret_cast<SpSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort_flag = &sm->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int MT = (O + sp::BM - 1) / sp::BM;   // output-row tiles
    const int NT = (T + sp::BN - 1) / sp::BN;   // token tiles
    const int tiles = MT * NT;
    const int KB = (K + sp::BK - 1) / sp::BK;

    if (threadIdx.x == 32) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_y);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < sp::STAGES; ++s) {
            mbar_init(&sm->full_tma[s], 1);
            mbar_init(&sm->full_meta[s], sp::META_WARPS);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->tmem_full[b], 1);
            mbar_init(&sm->tmem_empty[b], sp::EPI_WARPS);
        }
        mbar_init(&sm->mma_done, 1);
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == sp::WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                     "r"(sp::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sm->tmem_base;
    asm volatile("griddepcontrol.wait;" ::: "memory");

    auto give_up = [&]() {
        if (!*abort_flag) {
            *abort_flag = 1;
            raise_status(status, kStatusTimeout);
        }
    };

    if (warp < sp::EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        // Thread (warp w, lane l) owns output row o = m0 + 32(w % 4) + l; per
        // slice of 32 tokens it holds acc[t, o] for those tokens and stores
        // y[t, o]: each store instruction of the warp writes 32 consecutive
        // outputs of one token.
        constexpr int NSL = sp::BN / 32;                 // slices per tile
        constexpr int MY = NSL / 2;                      // slices per warp
        const int quad = warp & 3, half = warp >> 2;
        auto run = [&](auto bf16_tag) {
            constexpr bool BF = decltype(bf16_tag)::value;
            using OutT = typename std::conditional<BF, __nv_bfloat16, float>::type;
            OutT* const yp = reinterpret_cast<OutT*>(y);
            const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
            int tc = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
                const int mt = tile % MT, nt = tile / MT;
                const int b = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                const int o = mt * sp::BM + quad * 32 + lane;
                const bool ovalid = o < O;
                const float sc = ovalid ? __ldg(row_scale + o) : 0.f;
                // token scales of this warp's slices, loaded before the accumulator wait
                float inv_my[MY];
#pragma unroll
                for (int jj = 0; jj < MY; ++jj) {
                    const int t = nt * sp::BN + 32 * (half + 2 * jj) + lane;
                    inv_my[jj] = t < T ? __ldg(s_tok + t) : 1.f;
                }
                if (!warp_wait(&sm->tmem_full[b], aph, abort_flag)) { give_up(); break; }
                tc_fence_after();
#pragma unroll
                for (int jj = 0; jj < MY; ++jj) inv_my[jj] = __frcp_rn(inv_my[jj]);
                const uint32_t tbase = tmem_base + lane_addr + b * sp::BN;
                uint32_t ra[32], rb[32];
                // slice number jj of this warp: columns 32 (half + 2 jj); `cur` holds
                // it, the next one loads into `nxt` meanwhile
                auto slice = [&](const int jj, uint32_t (&cur)[32], uint32_t (&nxt)[32]) {
                    if (jj + 1 < MY) {
                        tmem_ld32_nowait(tbase + 32 * (half + 2 * (jj + 1)), nxt);
                    } else {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm->tmem_empty[b]);  // the warp is done with the buffer
                    }
                    const int t0 = nt * sp::BN + 32 * (half + 2 * jj);
                    if (t0 < T) {
                        const float inv_l = inv_my[jj];
                        const int nt_valid = T - t0 < 32 ? T - t0 : 32;
                        if (y_vec) {
                            // transpose through the warp's box: row i = token t0 + i,
                            // column lane = output o; one TMA store writes the box and
                            // clips rows past T and columns past O
                            uint8_t* const box = sm->ybox[warp];
                            if (lane == 0) bulk_wait_read<0>();  // the previous store has read the box
                            __syncwarp();
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const float f = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(cur[i])), sc),
                                                          __shfl_sync(0xFFFFFFFFu, inv_l, i));
                                if constexpr (BF) {
                                    const __nv_bfloat16 h = __float2bfloat16_rn(f);
                                    *reinterpret_cast<__nv_bfloat16*>(box + i * 64 + lane * 2) = h;
                                } else {
                                    *reinterpret_cast<float*>(box + i * 128 + lane * 4) = f;
                                }
                            }
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) tma_store_2d(&tmap_y, smem_u32(box), mt * sp::BM + quad * 32, t0);
                        } else {
                            // direct stores: shapes whose row pitch is not a multiple of 16 bytes
                            OutT* p = yp + static_cast<long long>(t0) * O + o;
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const float inv_s = __shfl_sync(0xFFFFFFFFu, inv_l, i);
                                if (ovalid && i < nt_valid) {
                                    const float f =
                                        __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(cur[i])), sc), inv_s);
                                    if constexpr (BF) *p = __float2bfloat16_rn(f);
                                    else *p = f;
                                }
                                p += O;
                            }
                        }
                        if (acc_out && ovalid) {
                            int32_t* pa = acc_out + static_cast<long long>(t0) * O + o;
#pragma unroll
                            for (int i = 0; i < 32; ++i, pa += O)
                                if (i < nt_valid) *pa = static_cast<int>(cur[i]);
                        }
                    }
                    if (jj + 1 < MY) tmem_ld_wait();
                };
                tmem_ld32_nowait(tbase + 32 * half, ra);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < MY; jj += 2) {
                    slice(jj, ra, rb);
                    if (jj + 1 < MY) slice(jj + 1, rb, ra);
                }
            }
            if (lane == 0) bulk_wait_all();
        };
        if (y_bf16) run(std::true_type{});
        else run(std::false_type{});
    } else if (warp < sp::WARP_TMA) {
        // ------------------------------------------------------------ metadata into tensor memory
        // Warp WARP_META + q writes TMEM lanes 32q .. 32q + 31 (rows of the weight
        // tile).  The nibbles of a k-block are loaded two k-blocks ahead, so that
        // only the tensor-memory store waits for the stage to be free.
        const int q = warp - sp::WARP_META;
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const long long total = static_cast<long long>((tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                                       static_cast<int>(gridDim.x)) * KB;  // this CTA's k-blocks
        // the nibble words of this CTA's k-block number `it` for this thread's row
        auto fetch = [&](long long it, uint32_t (&v)[8]) {
            const int tile = static_cast<int>(blockIdx.x) + static_cast<int>(it / KB) * static_cast<int>(gridDim.x);
            const int kb = static_cast<int>(it % KB);
            const int row = (tile % MT) * sp::BM + q * 32 + lane;
            if (it < total && row < O) {
                const uint8_t* src = meta + static_cast<long long>(row) * e_pitch + kb * sp::E_BYTES_ROW;
                const uint4 lo = ldg_nc(src);
                const uint4 hi = ldg_nc(src + 16);
                v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
                v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0u;
            }
        };
        uint32_t v0[8], v1[8], v2[8];
        fetch(0, v0);
        fetch(1, v1);
        for (long long it = 0; it < total; ++it) {
            fetch(it + 2, v2);
            const int s = static_cast<int>(it % sp::STAGES);
            const uint32_t ph = static_cast<uint32_t>(it / sp::STAGES) & 1u;
            // the stage's MMAs are done with its metadata columns
            if (!warp_wait(&sm->empty[s], ph ^ 1, abort_flag)) { give_up(); break; }
            tmem_st8(tmem_base + lane_addr + sp::E_COL0 + s * (sp::BK / 32), v0);
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->full_meta[s]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v0[i] = v1[i];
                v1[i] = v2[i];
            }
        }
    } else if (warp == sp::WARP_TMA) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int mt = tile % MT, nt = tile / MT;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % sp::STAGES;
                    const uint32_t ph = (it / sp::STAGES) & 1;
                    if (!mbar_wait(&sm->empty[s], ph ^ 1, abort_flag)) { give_up(); ok = false; break; }
                    mbar_arrive_expect_tx(&sm->full_tma[s], sp::A_BYTES + sp::B_BYTES);
                    tma_load_2d(smem_u32(sm->a[s]), &tmap_a, kb * (sp::BK / 2), mt * sp::BM, &sm->full_tma[s]);
                    tma_load_2d(smem_u32(sm->b[s]), &tmap_x, kb * sp::BK, nt * sp::BN, &sm->full_tma[s]);
                    tma_load_2d(smem_u32(sm->b[s] + sp::B_HALF), &tmap_x, kb * sp::BK + 128, nt * sp::BN,
                                &sm->full_tma[s]);
                }
            }
            const uint32_t first = it > sp::STAGES ? it - sp::STAGES : 0;
            volatile int never = 0;
            for (uint32_t j = first; j < it; ++j)
                if (!mbar_wait(&sm->full_tma[j % sp::STAGES], (j / sp::STAGES) & 1, &never)) give_up();
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = sp_idesc();
            uint32_t it = 0;
            int tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
                const int b = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                if (!mbar_wait(&sm->tmem_empty[b], aph ^ 1, abort_flag)) { give_up(); break; }
                tc_fence_after();
                const uint32_t d = tmem_base + b * sp::BN;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % sp::STAGES;
                    const uint32_t ph = (it / sp::STAGES) & 1;
                    if (!mbar_wait(&sm->full_tma[s], ph, abort_flag) || !mbar_wait(&sm->full_meta[s], ph, abort_flag)) {
                        give_up(); ok = false; break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sm->a[s]), b0 = smem_u32(sm->b[s]);
                    const uint32_t e0 = tmem_base + sp::E_COL0 + s * (sp::BK / 32);
#pragma unroll
                    for (int kk = 0; kk < sp::BK / 64; ++kk)
                        tc_mma_sp(d, sw128_desc(a0 + kk * 32), sw128_desc(b0 + (kk >> 1) * sp::B_HALF + (kk & 1) * 64),
                                  e0 + 2 * kk, idesc, (kb | kk) != 0);
                    tc_commit(&sm->empty[s]);
                }
                if (ok) tc_commit(&sm->tmem_full[b]);
            }
            tc_commit(&sm->mma_done);
            volatile int never = 0;
            if (!mbar_wait(&sm->mma_done, 0, &never)) give_up();
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == sp::WARP_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(sp::TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// host side
size_t sp_scratch_bytes(long long O, long long K) {
    const auto r256 = [](size_t b) { return (b + 255) & ~static_cast<size_t>(255); };
    return r256(static_cast<size_t>(O) * static_cast<size_t>(sp_values_pitch(K))) +
           r256(static_cast<size_t>(O) * static_cast<size_t>(sp_meta_pitch(K)));
}

cudaError_t launch_prefill_sp(const int8_t* xq, const float* s_tok, long long T, long long K, const uint8_t* packed,
                              const float* row_scale, long long O, void* y, int y_bf16, int32_t* acc_out,
                              uint8_t* scratch, unsigned* status, int num_sms, cudaStream_t stream) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    uint8_t* values = scratch;
    const size_t vbytes = (static_cast<size_t>(O) * static_cast<size_t>(sp_values_pitch(K)) + 255) & ~static_cast<size_t>(255);
    uint8_t* meta = scratch + vbytes;
    const long long e_pitch = sp_meta_pitch(K);
    {
        const long long work = O * (e_pitch / 2);
        long long blocks = (work + 255) / 256;
        if (blocks > 8LL * num_sms) blocks = 8LL * num_sms;
        sp_compress_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            reinterpret_cast<const uint32_t*>(packed), O, K, reinterpret_cast<uint16_t*>(values), meta, status);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap map_a, map_x;
    const cuuint32_t estr[2] = {1, 1};
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(O)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(sp::BK / 2), static_cast<cuuint32_t>(sp::BM)};
        if (enc(&map_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, values, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
        const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(sp::BN)};
        if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(xq), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    // output boxes of 32 tokens x 32 outputs go out by TMA when the row pitch allows it
    const int esize = y_bf16 ? 2 : 4;
    int y_vec = (O * esize) % 16 == 0 ? 1 : 0;
    CUtensorMap map_y = map_x;
    if (y_vec) {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(O), static_cast<cuuint64_t>(T)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(O) * esize};
        const cuuint32_t box[2] = {32u, 32u};
        if (enc(&map_y, y_bf16 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, y, dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            y_vec = 0;
    }
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_sp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(sp_smem_bytes()));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const long long tiles = ((O + sp::BM - 1) / sp::BM) * ((T + sp::BN - 1) / sp::BN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(sp::THREADS);
    cfg.dynamicSmemBytes = sp_smem_bytes();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_sp_kernel, map_a, map_x, map_y, y_vec, static_cast<const uint8_t*>(meta), e_pitch,
                              row_scale, s_tok, static_cast<int>(T), static_cast<int>(O), static_cast<int>(K), y,
                              y_bf16, acc_out, status);
}

}  // namespace sbl
