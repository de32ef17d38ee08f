// Mask change rate and mask verification between two N:M mask bitmaps.
//
// Training rebuilds the mask as the latent weights move; the Sparse-BitNet
// README ("Features": dynamic mask monitoring, with a CLI interval for the
// mask change rate) and the halo-sparse-bitnet-3:4-500m card ("Recipe":
// mask-verify every 500 steps) watch two statistics, computed here in one
// pass over two bitmaps (uint8 [O, K/8], bit k % 8 of byte k / 8 = weight k
// kept, the layout sbl_prepare_weights writes):
//   changed     positions whose kept state differs (popcount of old XOR new),
//               in total and per row;
//   bad groups  M-groups of the new mask that do not keep exactly N weights
//               (M = 4: a nibble, M = 8: a byte, counted with bit-sliced
//               popcounts of all groups of a 32-bit word at once).
// One warp per row, words of 16, 4 or 2 bytes as the row pitch allows; the
// block sums its warps' counts and adds them to the totals with one 64-bit
// atomic each.  HBM-bound: 2 * O * K / 8 bytes read.
#include "sbl_common.cuh"

namespace sbl {

constexpr int kMonWarps = 8;

// M-groups of `v` (bits of `valid` mark the groups that exist) whose kept count is not n.
template <int M>
__device__ __forceinline__ uint32_t bad_groups(uint32_t v, uint32_t n_rep, uint32_t valid) {
    uint32_t c = v - ((v >> 1) & 0x55555555u);
    c = (c & 0x33333333u) + ((c >> 2) & 0x33333333u);  // kept count of each nibble
    if constexpr (M == 4) {
        const uint32_t x = c ^ n_rep;                     // nonzero nibble: count != n (values < 8)
        return __popc((x | (x >> 1) | (x >> 2)) & 0x11111111u & valid);
    } else {
        c = (c + (c >> 4)) & 0x0F0F0F0Fu;                 // kept count of each byte
        const uint32_t x = c ^ n_rep;                     // values < 16
        return __popc((x | (x >> 1) | (x >> 2) | (x >> 3)) & 0x01010101u & valid);
    }
}

template <int M, typename Word>
__global__ void __launch_bounds__(kMonWarps * 32) mask_monitor_kernel(const uint8_t* __restrict__ old_bits,
                                                                      const uint8_t* __restrict__ new_bits,
                                                                      long long O, int row_bytes, int n,
                                                                      unsigned long long* __restrict__ totals,
                                                                      uint32_t* __restrict__ row_changed) {
    __shared__ unsigned long long part[2][kMonWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * kMonWarps + warp;
    uint32_t changed = 0, bad = 0;
    if (row < O) {
        constexpr int WB = sizeof(Word);
        constexpr int PARTS = WB >= 4 ? WB / 4 : 1;  // 32-bit pieces per word
        const uint32_t n_rep = M == 4 ? static_cast<uint32_t>(n) * 0x11111111u : static_cast<uint32_t>(n) * 0x01010101u;
        // a 2-byte word fills the low half of its piece: only the groups there exist
        const uint32_t valid = WB >= 4 ? 0xFFFFFFFFu : 0x0000FFFFu;
        const Word* a = reinterpret_cast<const Word*>(old_bits + row * row_bytes);
        const Word* b = reinterpret_cast<const Word*>(new_bits + row * row_bytes);
        const int nw = row_bytes / WB;
        for (int i = lane; i < nw; i += 32) {
            const Word wa = __ldg(a + i), wb = __ldg(b + i);
            uint32_t pa[PARTS], pb[PARTS];
            if constexpr (WB == 16) {
                pa[0] = wa.x; pa[1 % PARTS] = wa.y; pa[2 % PARTS] = wa.z; pa[3 % PARTS] = wa.w;
                pb[0] = wb.x; pb[1 % PARTS] = wb.y; pb[2 % PARTS] = wb.z; pb[3 % PARTS] = wb.w;
            } else {
                pa[0] = static_cast<uint32_t>(wa);
                pb[0] = static_cast<uint32_t>(wb);
            }
#pragma unroll
            for (int p = 0; p < PARTS; ++p) {
                changed += __popc(pa[p] ^ pb[p]);
                bad += bad_groups<M>(pb[p], n_rep, valid);
            }
        }
        changed = __reduce_add_sync(0xFFFFFFFFu, changed);
        bad = __reduce_add_sync(0xFFFFFFFFu, bad);
        if (lane == 0 && row_changed) row_changed[row] = changed;
    }
    if (lane == 0) {
        part[0][warp] = changed;
        part[1][warp] = bad;
    }
    __syncthreads();
    if (threadIdx.x < 2) {
        unsigned long long s = 0;
#pragma unroll
        for (int w = 0; w < kMonWarps; ++w) s += part[threadIdx.x][w];
        if (s) atomicAdd(totals + threadIdx.x, s);
    }
}

template <int M>
static cudaError_t launch_mon_m(const uint8_t* old_bits, const uint8_t* new_bits, long long O, long long K, int n,
                                unsigned long long* totals, uint32_t* row_changed, cudaStream_t stream) {
    const int row_bytes = static_cast<int>(K / 8);
    const unsigned blocks = static_cast<unsigned>((O + kMonWarps - 1) / kMonWarps);
    if (row_bytes % 16 == 0)
        mask_monitor_kernel<M, uint4><<<blocks, kMonWarps * 32, 0, stream>>>(old_bits, new_bits, O, row_bytes, n,
                                                                             totals, row_changed);
    else if (row_bytes % 4 == 0)
        mask_monitor_kernel<M, uint32_t><<<blocks, kMonWarps * 32, 0, stream>>>(old_bits, new_bits, O, row_bytes, n,
                                                                                totals, row_changed);
    else
        mask_monitor_kernel<M, uint16_t><<<blocks, kMonWarps * 32, 0, stream>>>(old_bits, new_bits, O, row_bytes, n,
                                                                                totals, row_changed);
    return cudaGetLastError();
}

// totals[0] = changed positions, totals[1] = bad groups (zeroed here first);
// row_changed [O] may be null.  Needs K % 16 == 0 and 16-byte aligned bitmaps.
cudaError_t launch_mask_monitor(const uint8_t* old_bits, const uint8_t* new_bits, long long O, long long K, int n,
                                int m, unsigned long long* totals, uint32_t* row_changed, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(totals, 0, 2 * sizeof(unsigned long long), stream);
    if (e != cudaSuccess) return e;
    return m == 4 ? launch_mon_m<4>(old_bits, new_bits, O, K, n, totals, row_changed, stream)
                  : launch_mon_m<8>(old_bits, new_bits, O, K, n, totals, row_changed, stream);
}

}  // namespace sbl
