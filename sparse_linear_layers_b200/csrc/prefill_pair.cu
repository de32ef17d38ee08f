// Prefill path on CTA pairs: acc[t, o] = sum_k x_q[t, k] * W_t[o, k] with
// 2-SM tcgen05 MMAs (cta_group::2, kind::i8), then y = acc * scale_o / s_t.
//
// The contraction of the Sparse-BitNet Guide's linear-evaluation equation
// ("Mathematical Formulation of Sparse-BitLinear"), for many tokens a dense
// int8 matrix product.  A cluster of two CTAs (on two SMs) computes one
// 256-token x 256-output tile per step of its persistent loop:
//
//   CTA rank r holds tokens 128r .. 128r + 127 of the tile (its half of A),
//   output rows 128r .. 128r + 127 (its half of B: 2-bit codes loaded by TMA
//   and expanded to int8 in its own shared memory) and, in its own tensor
//   memory, the accumulators of its 128 tokens for all 256 outputs.  The
//   even CTA issues the MMAs (M = 256, N = 256, K = 32), which read both
//   CTAs' shared memory.
//
// Against one CTA computing a 128 x 256 tile, each SM now expands and stores
// half as many weight bytes and its shared memory delivers half of B per MMA
// instead of all of it; per 128-deep k-block an SM moves about 72 KB of
// shared-memory traffic (activation tile written by TMA and read by the MMA,
// code tile written and read, int8 weight half written and read) for the
// same 128 x 256 x 128 multiply-adds that cost about 112 KB on one CTA.
//
// Warp roles in each CTA (448 threads):
//   warps 0-7  epilogue: warp w owns TMEM lanes 32 (w % 4) .. + 31 (32 tokens)
//              and accumulator columns 128 (w / 4) .. + 127; pipelined
//              tcgen05.ld, dequantise, a 128B-swizzled staging box, TMA bulk
//              stores (with four warps the fp32 epilogue of a 256 x 256 tile,
//              128 KB per CTA, outlasted the tile's MMAs at K = 896)
//   warps 8-11 weight expansion: one thread per output row of the CTA's half
//   warp 12    TMA producer (activation half-tile, code half-tile)
//   warp 13    TMEM allocation (both CTAs) and, in the even CTA, MMA issue
//
// Barriers: the activation loads of both CTAs complete on the even CTA's
// full_a; each CTA's code tile completes on its own full_c; the expansion
// threads of both CTAs arrive on the even CTA's full_dec; MMA completion is
// committed to empty / tmem_full / mma_done in both CTAs at once; the
// epilogue threads of both CTAs arrive on the even CTA's tmem_empty.  Every
// wait is bounded; a CTA that gives up records a timeout and winds down.
#include <cuda.h>

#include <cstring>
#include <type_traits>

#include "sbl_common.cuh"
#include "tc_util.cuh"

namespace sbl {

#ifdef SBL_TRACE
// Debug builds only: clock64 stamps of pipeline events in CTA 0 (the even CTA
// of the first pair): event e, iteration i -> g_trace_pair[e * 256 + i].
__device__ unsigned long long* g_trace_pair;
#define SBLP_TR(e, i)                                                            \
    do {                                                                         \
        if (trace_buf && (i) < 256) trace_buf[(e) * 256 + (i)] = clock64();     \
    } while (0)
#else
#define SBLP_TR(e, i) \
    do {              \
    } while (0)
#endif

namespace pp {
constexpr int BM = 128;                     // tokens per CTA (pair: 256)
constexpr int BN = 256;                     // outputs per pair tile
constexpr int BNH = BN / 2;                 // output rows held by one CTA
constexpr int BK = 128;                     // k per stage (bytes of int8)
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BNH * BK;
constexpr int P_BYTES = BNH * BK / 4;       // 2-bit codes of the CTA's half of B
constexpr int STAGES = 5;
constexpr int EPI_WARPS = 8;              // two per TMEM lane quadrant, one per column half
constexpr int DEC_WARPS = BNH / 32;
constexpr int WARP_TMA = EPI_WARPS + DEC_WARPS;
constexpr int WARP_MMA = WARP_TMA + 1;
constexpr int THREADS = (WARP_MMA + 1) * 32;
constexpr int TMEM_COLS = 2 * BN;           // two accumulator buffers
constexpr int Y_BYTES = 32 * 128;           // one warp's staging box: 32 tokens x 128 bytes
}  // namespace pp

struct PairSmem {
    uint8_t a[pp::STAGES][pp::A_BYTES];     // 1024-byte aligned tiles
    uint8_t b[pp::STAGES][pp::B_BYTES];
    uint8_t p[pp::STAGES][pp::P_BYTES];
    uint8_t ystage[pp::EPI_WARPS][pp::Y_BYTES];    // one staging box per epilogue warp
    float wscale[pp::EPI_WARPS][pp::BN / 2];
    uint64_t full_a[pp::STAGES];            // used in the even CTA
    uint64_t full_c[pp::STAGES];
    uint64_t full_dec[pp::STAGES];          // used in the even CTA
    uint64_t empty[pp::STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];                 // used in the even CTA
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t pair_smem_bytes() { return sizeof(PairSmem) + 1024; }
static_assert(pair_smem_bytes() <= 232448, "pair prefill tile does not fit in shared memory");

template <bool GROUPED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pp::THREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ PrefillOut out,
                        const float* __restrict__ s_tok, int T, int K, int y_bf16, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    auto* sm = reinterpret_cast<PairSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort_flag = &sm->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#ifdef SBL_TRACE
    unsigned long long* const trace_buf = blockIdx.x == 0 ? g_trace_pair : nullptr;
#endif
    if (threadIdx.x == 0) SBLP_TR(8, 0);  // entry
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int MT = (T + 2 * pp::BM - 1) / (2 * pp::BM);
    const int NT = GROUPED ? out.nt_end[out.G - 1] : out.nt_end[0];  // output tiles of all layers
    const int tiles = MT * NT;
    const int KB = (K + pp::BK - 1) / pp::BK;

    if (threadIdx.x == 32) {
        prefetch_tmap(&tmap_x);
#pragma unroll
        for (int i = 0; i < (GROUPED ? kPrefillMaxGroup : 1); ++i)
            if (i < out.G) {
                prefetch_tmap(&out.tmap_w[i]);
                prefetch_tmap(&out.tmap_y[i]);
            }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < pp::STAGES; ++s) {
            mbar_init(&sm->full_a[s], 1);
            mbar_init(&sm->full_c[s], 1);
            mbar_init(&sm->full_dec[s], 2 * pp::DEC_WARPS);  // one arrival per expansion warp
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->tmem_full[b], 1);
            mbar_init(&sm->tmem_empty[b], 2 * pp::EPI_WARPS);  // one arrival per epilogue warp
        }
        mbar_init(&sm->mma_done, 1);
        sm->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == pp::WARP_MMA) {
        // the same warp of both CTAs, the same destination offset
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                     "r"(pp::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = sm->tmem_base;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) SBLP_TR(9, 0);  // inputs visible

    auto give_up = [&]() {
        if (!*abort_flag) {
            *abort_flag = 1;
            raise_status(status, kStatusTimeout);
        }
    };
    // arrive on the even CTA's copy of a barrier
    auto arrive_leader = [&](uint64_t* bar) {
        if (leader) mbar_arrive(bar);
        else mbar_arrive_cluster(map_to_cta(smem_u32(bar), 0));
    };

    if (warp < pp::EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        // Warp w reads TMEM lanes 32 (w % 4) .. + 31 (32 tokens of the CTA's
        // half) and the 128 accumulator columns of half w / 4.  Per tile it
        // copies its 128 row scales into its shared-memory slice, waits for the
        // accumulator, then walks its four 32-column TMEM slices with the next
        // one in flight, dequantises and stores 128 output bytes per token per
        // round through its staging box.  Once all eight warps of both CTAs have
        // read the buffer it goes back to the even CTA's MMA issuer.
        auto run = [&](auto bf16_tag) {
            constexpr bool BF = decltype(bf16_tag)::value;
            constexpr int SPR = BF ? 2 : 1;          // 32-column slices per round
            constexpr int NSL = pp::BN / 64;         // slices of this warp per tile
            const int qd = warp & 3, half = warp >> 2;
            const int row = qd * 32 + lane;          // TMEM lane == token within the CTA's half
            const uint32_t lane_addr = static_cast<uint32_t>(qd * 32) << 16;
            const int col0 = half * (pp::BN / 2);    // first accumulator column of this warp
            float* const wsc = sm->wscale[warp];
            int tc = 0;
            for (int tile = pair; tile < tiles; tile += npairs, ++tc) {
                const int mt = tile / NT;  // output tiles fastest: a token tile is read once
                int g = 0, nt = tile % NT;
                if (GROUPED) {
                    while (g + 1 < out.G && nt >= out.nt_end[g]) ++g;
                    if (g > 0) nt -= out.nt_end[g - 1];
                }
                const int O = out.O[g], y_vec = out.y_vec[g];
                const float* const row_scale = out.row_scale[g];
                const int b = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                __syncwarp();
#pragma unroll
                for (int k = 0; k < NSL; ++k) {
                    const int o = nt * pp::BN + col0 + 32 * k + lane;
                    wsc[32 * k + lane] = o < O ? __ldg(row_scale + o) : 0.f;
                }
                __syncwarp();
                if (!warp_wait(&sm->tmem_full[b], aph, abort_flag)) { give_up(); break; }
                if (lane == 0 && warp == 0) SBLP_TR(5, tc);
                if (lane == 0 && warp == 4) SBLP_TR(7, tc);
                tc_fence_after();
                const int trow0 = mt * 2 * pp::BM + static_cast<int>(rank) * pp::BM;
                const int t = trow0 + row;
                const bool tvalid = t < T;
                const float inv_s = tvalid ? __frcp_rn(s_tok[t]) : 0.f;
                const uint32_t tbase = tmem_base + lane_addr + b * pp::BN + col0;
                uint32_t ra[32], rb[32];
                auto slice = [&](auto h_tag, const int k, uint32_t (&cur)[32], uint32_t (&nxt)[32]) {
                    constexpr int H = decltype(h_tag)::value;
                    const bool more = k + 1 < NSL;
                    if (more) {
                        tmem_ld32_nowait(tbase + 32 * (k + 1), nxt);
                    } else {
                        // the warp is done with the buffer (its loads completed above)
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) arrive_leader(&sm->tmem_empty[b]);
                        if (lane == 0 && warp == 0) SBLP_TR(6, tc);
                    }
                    const float* sc = wsc + 32 * k;
                    const int o0 = nt * pp::BN + col0 + 32 * (k - H);  // first output of the round
                    uint8_t* const box = sm->ystage[warp];
                    if (y_vec && H == 0) {
                        if (lane == 0) bulk_wait_read<0>();  // the box's previous store has read it
                        __syncwarp();
                    }
                    // 16 output bytes at a time: into the lane's row of the staging
                    // box (128B-swizzled) or, for shapes whose row pitch is not a
                    // multiple of 16 bytes, straight to y
                    auto put = [&](const int c, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
                        if (y_vec) {
                            const uint32_t a = smem_u32(box + lane * 128 + ((c ^ (lane & 7)) << 4));
                            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(w0), "r"(w1), "r"(w2),
                                         "r"(w3)
                                         : "memory");
                        } else if (tvalid) {
                            void* const y = out.y[g];
                            const long long base = static_cast<long long>(t) * O + o0;
                            const uint32_t w[4] = {w0, w1, w2, w3};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                if (BF) {
                                    const int e = 8 * c + 2 * j;
                                    if (o0 + e < O) reinterpret_cast<uint16_t*>(y)[base + e] = static_cast<uint16_t>(w[j] & 0xFFFFu);
                                    if (o0 + e + 1 < O) reinterpret_cast<uint16_t*>(y)[base + e + 1] = static_cast<uint16_t>(w[j] >> 16);
                                } else {
                                    const int e = 4 * c + j;
                                    if (o0 + e < O) reinterpret_cast<uint32_t*>(y)[base + e] = w[j];
                                }
                            }
                        }
                    };
                    auto deq = [&](int i) {  // y of column i of the slice, before the output rounding
                        return __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(cur[i])), sc[i]), inv_s);
                    };
                    if (BF) {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {  // 8 columns per 16-byte chunk
                            const int i = 8 * c;
                            const __nv_bfloat162 h0 = __floats2bfloat162_rn(deq(i), deq(i + 1));
                            const __nv_bfloat162 h1 = __floats2bfloat162_rn(deq(i + 2), deq(i + 3));
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(deq(i + 4), deq(i + 5));
                            const __nv_bfloat162 h3 = __floats2bfloat162_rn(deq(i + 6), deq(i + 7));
                            put(4 * H + c, *reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                                *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c) {  // 4 columns per 16-byte chunk
                            const int i = 4 * c;
                            put(c, __float_as_uint(deq(i)), __float_as_uint(deq(i + 1)), __float_as_uint(deq(i + 2)),
                                __float_as_uint(deq(i + 3)));
                        }
                    }
                    int32_t* const acc_out = out.acc_out[g];
                    if (acc_out && tvalid) {
                        const long long base = static_cast<long long>(t) * O + nt * pp::BN + col0 + 32 * k;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (nt * pp::BN + col0 + 32 * k + i < O) acc_out[base + i] = static_cast<int>(cur[i]);
                    }
                    if (H == SPR - 1 && y_vec) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0)
                            tma_store_2d(tile_owner<GROUPED>(out, tile % NT).tmap_y, smem_u32(box), o0, trow0 + qd * 32);
                    }
                    if (more) tmem_ld_wait();
                };
                tmem_ld32_nowait(tbase, ra);
                tmem_ld_wait();
                for (int k = 0; k < NSL; k += 2) {
                    if (SPR == 2) {
                        slice(std::integral_constant<int, 0>{}, k, ra, rb);
                        slice(std::integral_constant<int, 1>{}, k + 1, rb, ra);
                    } else {
                        slice(std::integral_constant<int, 0>{}, k, ra, rb);
                        slice(std::integral_constant<int, 0>{}, k + 1, rb, ra);
                    }
                }
            }
            if (lane == 0) bulk_wait_all();
        };
        if (y_bf16) run(std::true_type{});
        else run(std::false_type{});
    } else if (warp < pp::WARP_TMA) {
        // ------------------------------------------------------------ weight expansion
        // Thread r expands output row r of this CTA's half of B for each k-block
        // and reports to the even CTA, whose MMAs read this shared memory.
        const int r = threadIdx.x - pp::EPI_WARPS * 32;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = pair; tile < tiles && ok; tile += npairs) {
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % pp::STAGES;
                const uint32_t ph = (it / pp::STAGES) & 1;
                // the codes have landed; the producer loaded them only after the
                // pair's MMAs released this stage, so b[s] is free as well
                if (!mbar_wait(&sm->full_c[s], ph, abort_flag)) { give_up(); ok = false; break; }
                if (r == 0) SBLP_TR(1, it);
                // code rows are 32 bytes, 32B-swizzled by TMA: 16-byte half q of
                // row r sits at half q ^ ((r >> 2) & 1)
                const uint8_t* src = sm->p[s] + r * 32;
                const int hs = (r >> 2) & 1;
                const uint4 p0 = *reinterpret_cast<const uint4*>(src + (hs << 4));
                const uint4 p1 = *reinterpret_cast<const uint4*>(src + ((hs ^ 1) << 4));
                uint8_t* dst = sm->b[s] + r * 128;
                const int sw = r & 7;
                const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t e[4];
                    expand_pairs(words[c], e);
                    const uint32_t a = smem_u32(dst + ((c ^ sw) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(e[0]), "r"(e[1]), "r"(e[2]),
                                 "r"(e[3])
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if ((r & 31) == 0) arrive_leader(&sm->full_dec[s]);
                if (r == 0) SBLP_TR(2, it);
            }
        }
    } else if (warp == pp::WARP_TMA) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = pair; tile < tiles && ok; tile += npairs) {
                const int mt = tile / NT;  // output tiles fastest: a token tile is read once
                const TileOwner own = tile_owner<GROUPED>(out, tile % NT);
                const int trow = mt * 2 * pp::BM + static_cast<int>(rank) * pp::BM;
                const int orow = own.nt * pp::BN + static_cast<int>(rank) * pp::BNH;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % pp::STAGES;
                    const uint32_t ph = (it / pp::STAGES) & 1;
                    if (!mbar_wait(&sm->empty[s], ph ^ 1, abort_flag)) { give_up(); ok = false; break; }
                    SBLP_TR(0, it);
                    // the even CTA expects the activation bytes of both CTAs
                    if (leader) mbar_arrive_expect_tx(&sm->full_a[s], 2 * pp::A_BYTES);
                    mbar_arrive_expect_tx(&sm->full_c[s], pp::P_BYTES);
                    tma_load_2d_pair(smem_u32(sm->a[s]), &tmap_x, kb * pp::BK, trow,
                                     map_to_cta(smem_u32(&sm->full_a[s]), 0));
                    tma_load_2d(smem_u32(sm->p[s]), own.tmap_w, kb * (pp::BK / 4), orow, &sm->full_c[s]);
                }
            }
            // let the issued loads land before the CTA can exit: its own code
            // tiles here, and (in the even CTA) the activation tiles of both
            const uint32_t first = it > pp::STAGES ? it - pp::STAGES : 0;
            volatile int never = 0;
            for (uint32_t j = first; j < it; ++j) {
                const int s = j % pp::STAGES;
                const uint32_t ph = (j / pp::STAGES) & 1;
                if (!mbar_wait(&sm->full_c[s], ph, &never)) give_up();
                if (leader && !mbar_wait(&sm->full_a[s], ph, &never)) give_up();
            }
        }
    } else {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0) {
            if (leader) {
                const uint32_t idesc = i8_idesc<2 * pp::BM, pp::BN>();
                uint32_t it = 0;
                int tc = 0;
                bool ok = true;
                for (int tile = pair; tile < tiles && ok; tile += npairs, ++tc) {
                    const int b = tc & 1;
                    const uint32_t aph = (tc >> 1) & 1;
                    if (!mbar_wait(&sm->tmem_empty[b], aph ^ 1, abort_flag)) { give_up(); break; }
                    SBLP_TR(4, tc);
                    tc_fence_after();
                    const uint32_t d = tmem_base + b * pp::BN;
                    for (int kb = 0; kb < KB; ++kb, ++it) {
                        const int s = it % pp::STAGES;
                        const uint32_t ph = (it / pp::STAGES) & 1;
                        if (!mbar_wait(&sm->full_a[s], ph, abort_flag) ||
                            !mbar_wait(&sm->full_dec[s], ph, abort_flag)) {
                            give_up(); ok = false; break;
                        }
                        SBLP_TR(3, it);
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(sm->a[s]), b0 = smem_u32(sm->b[s]);
#pragma unroll
                        for (int kk = 0; kk < pp::BK / 32; ++kk)
                            tc_mma_pair(d, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc, (kb | kk) != 0);
                        tc_commit_pair_both(&sm->empty[s]);
                    }
                    if (ok) tc_commit_pair_both(&sm->tmem_full[b]);
                }
                // every MMA must be complete before either CTA frees tensor memory
                tc_commit_pair_both(&sm->mma_done);
            }
            volatile int never = 0;
            if (!mbar_wait(&sm->mma_done, 0, &never)) give_up();
        }
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync();  // neither CTA leaves while the other may still touch its shared memory
    if (warp == pp::WARP_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(pp::TMEM_COLS)
                     : "memory");
    }
}

// Opt the kernel in to its dynamic shared memory (once per device).
static cudaError_t pair_set_smem_attr() {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && attr_set[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(prefill_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(pair_smem_bytes()));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(pair_smem_bytes()));
    if (e == cudaSuccess && dev >= 0 && dev < 64) attr_set[dev] = true;
    return e;
}

// Clusters of this kernel that fit on the device at once (one CTA per SM, two
// SMs per cluster), cached per device; 0 when the query fails.
int prefill_pair_clusters(cudaStream_t stream) {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cached[dev] == 0) {
        if (pair_set_smem_attr() != cudaSuccess) return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(pp::THREADS);
        cfg.dynamicSmemBytes = pair_smem_bytes();
        cfg.stream = stream;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, prefill_pair_kernel<true>, &cfg) != cudaSuccess || n <= 0) return 0;
        cached[dev] = n;
    }
    return cached[dev];
}

// G layers (1 <= G <= kPrefillMaxGroup) that read the same quantised
// activations, in one launch of the CTA-pair kernel.
cudaError_t launch_prefill_pair_group(const int8_t* xperm, const float* s_tok, long long T, long long K, int G,
                                      const uint8_t* const* packed, const float* const* row_scale,
                                      const long long* O, void* const* y, int y_bf16, int32_t* const* acc_out,
                                      unsigned* status, cudaStream_t stream) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    if (G < 1 || G > kPrefillMaxGroup) return cudaErrorInvalidValue;
    if (cudaError_t e = pair_set_smem_attr()) return e;
    const int max_clusters = prefill_pair_clusters(stream);
    if (max_clusters <= 0) return cudaErrorNotSupported;

    CUtensorMap map_x;
    const cuuint32_t estr[2] = {1, 1};
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(pp::BK), static_cast<cuuint32_t>(pp::BM)};
        if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(xperm), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    PrefillOut out;
    memset(&out, 0, sizeof(out));
    out.G = G;
    int nt_end = 0;
    for (int g = 0; g < G; ++g) {
        {
            const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 4), static_cast<cuuint64_t>(O[g])};
            const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 4)};
            const cuuint32_t box[2] = {static_cast<cuuint32_t>(pp::BK / 4), static_cast<cuuint32_t>(pp::BNH)};
            if (enc(&out.tmap_w[g], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed[g]), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        const int esize = y_bf16 ? 2 : 4;
        out.y_vec[g] = (static_cast<long long>(O[g]) * esize) % 16 == 0 ? 1 : 0;
        out.tmap_y[g] = map_x;
        if (out.y_vec[g]) {
            const cuuint64_t dims[2] = {static_cast<cuuint64_t>(O[g]), static_cast<cuuint64_t>(T)};
            const cuuint64_t strides[1] = {static_cast<cuuint64_t>(O[g]) * esize};
            const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), 32u};
            if (enc(&out.tmap_y[g], y_bf16 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, y[g],
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                out.y_vec[g] = 0;
        }
        out.row_scale[g] = row_scale[g];
        out.y[g] = y[g];
        out.acc_out[g] = acc_out ? acc_out[g] : nullptr;
        out.O[g] = static_cast<int>(O[g]);
        nt_end += static_cast<int>((O[g] + pp::BN - 1) / pp::BN);
        out.nt_end[g] = nt_end;
    }
    const long long tiles = ((T + 2 * pp::BM - 1) / (2 * pp::BM)) * nt_end;
    const int clusters = static_cast<int>(tiles < max_clusters ? tiles : max_clusters);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(pp::THREADS);
    cfg.dynamicSmemBytes = pair_smem_bytes();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (G > 1)
        return cudaLaunchKernelEx(&cfg, prefill_pair_kernel<true>, map_x, out, s_tok, static_cast<int>(T),
                                  static_cast<int>(K), y_bf16, status);
    return cudaLaunchKernelEx(&cfg, prefill_pair_kernel<false>, map_x, out, s_tok, static_cast<int>(T),
                              static_cast<int>(K), y_bf16, status);
}

cudaError_t launch_prefill_pair(const int8_t* xperm, const float* s_tok, long long T, long long K,
                                const uint8_t* packed, const float* row_scale, long long O, void* y, int y_bf16,
                                int32_t* acc_out, unsigned* status, cudaStream_t stream) {
    void* yy[1] = {y};
    int32_t* aa[1] = {acc_out};
    return launch_prefill_pair_group(xperm, s_tok, T, K, 1, &packed, &row_scale, &O, yy, y_bf16, aa, status, stream);
}

#ifdef SBL_TRACE
cudaError_t set_pair_trace(void* buf) {
    unsigned long long* p = static_cast<unsigned long long*>(buf);
    return cudaMemcpyToSymbol(g_trace_pair, &p, sizeof(p));
}
#endif

}  // namespace sbl
