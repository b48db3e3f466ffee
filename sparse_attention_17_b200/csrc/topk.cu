// topk.cu -- exact top-k among the candidate lists of the filtered index selection
// (dsa_index_select): per-row thresholds from sampled scores, then the exact top-k among
// the keys the filtered indexer kept.  The dense per-row top-k is in topk_stream.cu.
//
// Selection rule (DSA ablation card, "Attention" bullet and closing note): the k largest
// of the row's n valid scores, equal scores resolved towards the lower key index; if
// n <= k every key is selected.  Output: the selected key positions in ascending order,
// then -1 padding.
//
// Scores map to order-preserving uint32 keys.  Each warp owns a slice of the shared
// candidate buffer, radix selection (12 + 12 + 8 bits) among the candidates gives the
// k-th largest key, and a bitmap of the selection is compacted in index order.
#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

constexpr int kBins = 4096;
constexpr int kCandCap = 8192;
constexpr int kBM_SAMPLE = 128;            // keys per sampled tile (the indexer's tile)
constexpr int kMaxWarps = 32;

// The block size of the candidate selection (512 threads, two CTAs per SM).
template <int T>
struct TopkCfg {
    static constexpr int kThreads = T;
    static constexpr int kWarps = T / 32;
    static constexpr int kSlice = kCandCap / kWarps;     // candidate entries of one warp
    static_assert(kWarps <= kMaxWarps && kSlice % 128 == 0, "block size");
};

struct TopkScratch {
    uint32_t hist[kBins];
    uint32_t cand_key[kCandCap];
    int cand_idx[kCandCap];
    uint32_t scan[kMaxWarps];
    uint32_t wcount[kMaxWarps];  // candidates appended by each warp (may exceed its slice)
    uint32_t cand_count;
    uint32_t found_bin;
    uint32_t found_above;
};

// Adds 1 to hist[bin] for every lane with pred, one shared atomic per distinct bin.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool pred) {
    const unsigned active = __ballot_sync(0xffffffffu, pred);
    if (pred) {
        const unsigned peers = __match_any_sync(active, bin);
        if ((int)lane_id() == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
}

// Exclusive prefix sum over the block's threads (in thread order); *total gets the sum.
template <int T>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, TopkScratch& sh,
                                                         uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh.scan[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < TopkCfg<T>::kWarps ? sh.scan[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < TopkCfg<T>::kWarps) sh.scan[lane] = w;
    }
    __syncthreads();
    const uint32_t before = (warp > 0 ? sh.scan[warp - 1] : 0u) + x - v;
    *total = sh.scan[TopkCfg<T>::kWarps - 1];
    __syncthreads();
    return before;
}

// Finds the bin b (scanning from the top) with above(b) < need <= above(b) + hist[b],
// above(b) = number of keys in bins higher than b.  Result in sh.found_bin/found_above.
template <int T>
__device__ void find_bin(TopkScratch& sh, int nbins, uint32_t need) {
    const int per = nbins >= TopkCfg<T>::kThreads ? nbins / TopkCfg<T>::kThreads : 1;
    const int first = nbins - 1 - (int)threadIdx.x * per;  // this thread's highest bin
    uint32_t local = 0;
    if (first >= 0)
        for (int i = 0; i < per; ++i) local += sh.hist[first - i];
    uint32_t total;
    uint32_t above = block_exclusive_scan<T>(local, sh, &total);
    if (first >= 0 && above < need && above + local >= need) {
        for (int i = 0; i < per; ++i) {
            const uint32_t c = sh.hist[first - i];
            if (above + c >= need) {
                sh.found_bin = (uint32_t)(first - i);
                sh.found_above = above;
                break;
            }
            above += c;
        }
    }
    __syncthreads();
}

template <int T>
__device__ __forceinline__ void zero_hist(TopkScratch& sh, int nbins) {
    for (int i = threadIdx.x; i < nbins; i += TopkCfg<T>::kThreads) sh.hist[i] = 0u;
}

// Radix select over the warps' candidate slices (warp w owns cand_key[w * TopkCfg<T>::kSlice ..] with
// wcount[w] <= TopkCfg<T>::kSlice entries).  exact: returns the need-th largest key tau and sets
// *need_out to how many keys equal to tau belong to the top `need` (12 + 12 + 8 bits).
// !exact: stops after 24 bits and returns the lower edge of the 24-bit bin holding the
// need-th largest key, a lower bound of it.
template <int T>
__device__ uint32_t slice_radix_select(TopkScratch& sh, uint32_t need, bool exact,
                                       uint32_t* need_out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t* keys = sh.cand_key + warp * TopkCfg<T>::kSlice;
    const int cnt = (int)sh.wcount[warp];
    zero_hist<T>(sh, kBins);
    __syncthreads();
    for (int c0 = 0; c0 < cnt; c0 += 32) {
        const int c = c0 + lane;
        hist_add(sh.hist, c < cnt ? keys[c] >> 20 : 0u, c < cnt);
    }
    __syncthreads();
    find_bin<T>(sh, kBins, need);
    const uint32_t b1 = sh.found_bin;
    need -= sh.found_above;
    zero_hist<T>(sh, kBins);
    __syncthreads();
    for (int c0 = 0; c0 < cnt; c0 += 32) {
        const int c = c0 + lane;
        const uint32_t key = c < cnt ? keys[c] : 0u;
        hist_add(sh.hist, (key >> 8) & 0xFFFu, c < cnt && (key >> 20) == b1);
    }
    __syncthreads();
    find_bin<T>(sh, kBins, need);
    const uint32_t pre = (b1 << 12) | sh.found_bin;
    need -= sh.found_above;
    if (!exact) {
        *need_out = need;
        __syncthreads();
        return pre << 8;
    }
    zero_hist<T>(sh, 256);
    __syncthreads();
    for (int c0 = 0; c0 < cnt; c0 += 32) {
        const int c = c0 + lane;
        const uint32_t key = c < cnt ? keys[c] : 0u;
        hist_add(sh.hist, key & 0xFFu, c < cnt && (key >> 8) == pre);
    }
    __syncthreads();
    find_bin<T>(sh, 256, need);
    need -= sh.found_above;
    *need_out = need;
    const uint32_t tau = (pre << 8) | sh.found_bin;
    __syncthreads();
    return tau;
}

// Keeps the first `need` ties (tie bitmap) in index order, merges them into the selection
// bitmap and writes the selected key positions in ascending order, then -1 up to k.
template <int T>
__device__ void trim_ties_and_compact(TopkScratch& sh, uint32_t* sel, const uint32_t* tie,
                                      int nwords, uint32_t need, int k, int* out,
                                      int idx_offset = 0) {
    const int wpt = (nwords + TopkCfg<T>::kThreads - 1) / TopkCfg<T>::kThreads;
    const int w0 = threadIdx.x * wpt;
    const int w1 = min(w0 + wpt, nwords);
    uint32_t local = 0;
    for (int w = w0; w < w1; ++w) local += __popc(tie[w]);
    uint32_t total;
    uint32_t before = block_exclusive_scan<T>(local, sh, &total);
    for (int w = w0; w < w1; ++w) {
        uint32_t tb = tie[w];
        const uint32_t c = __popc(tb);
        if (before >= need) {
            tb = 0u;
        } else if (before + c > need) {
            uint32_t keep = 0u, rest = tb;
            for (uint32_t m = need - before; m > 0; --m) {
                keep |= rest & (0u - rest);
                rest &= rest - 1u;
            }
            tb = keep;
        }
        before += c;
        sel[w] |= tb;
    }
    __syncthreads();
    local = 0;
    for (int w = w0; w < w1; ++w) local += __popc(sel[w]);
    uint32_t pos = block_exclusive_scan<T>(local, sh, &total);
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = sel[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1u;
            if (pos < (uint32_t)k) out[pos] = w * 32 + b + idx_offset;
            ++pos;
        }
    }
    for (int i = (int)total + threadIdx.x; i < k; i += TopkCfg<T>::kThreads) out[i] = -1;
}

// ---------------------------------------------------------------------------------------
// Filtered selection (no dense score rows): thresholds from sampled scores, then the exact
// top-k among the candidates the filtered indexer appended.
// ---------------------------------------------------------------------------------------
constexpr int kRowWarps = 8;          // rows per CTA of the warp-per-row kernels
constexpr int kSampleMax = 2048;      // sampled keys per row at most (64 per lane)

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One warp per row: tau[r] = the rank-th largest sampled order key, rank = e + 6 sqrt(e) + 2
// for the e = k * m / n samples expected above the row's k-th largest score.  The row's
// at most 2048 samples sit in registers (64 per lane) and the key is found bit by bit from
// the top: 32 counting passes of ballot-free compares and a warp sum, no shared memory.
// The first CTA also clears the window's fallback flag.
__global__ void __launch_bounds__(32 * kRowWarps)
topk_threshold_kernel(const float* __restrict__ sample, long long ld_sample, int q_begin,
                      int rows, int tile_stride, int k, uint32_t* __restrict__ tau,
                      int* __restrict__ fb_any) {
    constexpr int kPer = kSampleMax / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (blockIdx.x == 0 && threadIdx.x == 0) *fb_any = 0;
    const int r = blockIdx.x * kRowWarps + warp;
    if (r >= rows) return;
    const int t = q_begin + r;
    const int n = t + 1;
    // valid samples: logical tile j holds keys j*stride*128 .. +127, causal ones only
    const int span = kBM_SAMPLE * tile_stride;
    const int ntiles = t / span + 1;
    const int ncols = ntiles * kBM_SAMPLE;
    const int m = (ntiles - 1) * kBM_SAMPLE + min(kBM_SAMPLE, n - (ntiles - 1) * span);
    const float e = (float)k * (float)m / (float)n;
    uint32_t rank = (uint32_t)ceilf(e + 6.f * sqrtf(e)) + 2u;
    if (rank > (uint32_t)m) rank = (uint32_t)m;
    const float* row = sample + (long long)r * ld_sample;
    uint32_t key[kPer];  // 0 marks a missing sample (below every real order key)
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int c = i * 32 + lane;
        const bool in = c < ncols && (c / kBM_SAMPLE) * span + (c % kBM_SAMPLE) <= t;
        key[i] = in ? float_order_key(__ldg(row + c)) : 0u;
    }
    uint32_t prefix = 0u;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = prefix | (1u << bit);
        uint32_t cnt = 0;
#pragma unroll
        for (int i = 0; i < kPer; ++i) cnt += key[i] >= cand ? 1u : 0u;
        if (warp_sum(cnt) >= rank) prefix = cand;
    }
    if (lane == 0) tau[r] = prefix;
}

// One CTA per row: the exact top-k among the row's candidates (all keys at or above
// tau[r], kept in lists per 4096-key chunk and lane quadrant): with at least k of them the
// k-th largest key and every key equal to it are among them.  Rows whose lists overflowed
// or with fewer than k candidates are flagged for the dense fallback (fb_row[r] = 1,
// *fb_any = 1) and left unwritten.
template <int T>
__global__ void __launch_bounds__(T, T <= 512 ? 2 : 1)
topk_candidates_kernel(const uint2* __restrict__ cand, const uint32_t* __restrict__ ccount,
                       int cq, int nchunk_max, int q_begin, int max_len, int k,
                       int* __restrict__ idx, long long ld_idx, int* __restrict__ fb_row,
                       int* __restrict__ fb_any) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TopkScratch& sh = *reinterpret_cast<TopkScratch*>(smem_raw);
    uint32_t* sel = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkScratch));
    const int max_words = (max_len + 31) >> 5;
    uint32_t* tie = sel + max_words;

    const int r = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = q_begin + r + 1;
    int* out = idx + (long long)r * ld_idx;
    if (n <= k) {  // every valid key is selected
        if (threadIdx.x == 0) fb_row[r] = 0;
        for (int i = threadIdx.x; i < k; i += TopkCfg<T>::kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const int nwords = (n + 31) >> 5;
    for (int i = threadIdx.x; i < nwords; i += TopkCfg<T>::kThreads) sel[i] = 0u;
    // the row's lists (chunk, quadrant) are dealt round-robin to the warps, each appending
    // into its slice of the candidate buffer
    const int nlists = ((n + 4095) >> 12) * 4;
    const uint32_t* crow = ccount + (long long)r * nchunk_max * 4;
    const uint2* lrow = cand + (long long)r * nchunk_max * 4 * cq;
    uint32_t filled = 0;
    bool over = false;
    for (int l = warp; l < nlists; l += TopkCfg<T>::kWarps) {
        const uint32_t len = __ldg(crow + l);
        if (len > (uint32_t)cq || filled + len > (uint32_t)TopkCfg<T>::kSlice) { over = true; break; }
        const uint2* src = lrow + (long long)l * cq;
        for (uint32_t i = lane; i < len; i += 32) {
            const uint2 v = __ldg(src + i);
            sh.cand_key[warp * TopkCfg<T>::kSlice + filled + i] = v.x;
            sh.cand_idx[warp * TopkCfg<T>::kSlice + filled + i] = (int)v.y;
        }
        filled += len;
    }
    if (lane == 0) sh.wcount[warp] = over ? 0xFFFFFFFFu : filled;
    __syncthreads();
    uint32_t c = 0;
    bool fail = false;
#pragma unroll
    for (int w = 0; w < TopkCfg<T>::kWarps; ++w) {
        const uint32_t v = sh.wcount[w];
        fail |= v == 0xFFFFFFFFu;
        c += v;
    }
    if (fail || c < (uint32_t)k) {
        if (threadIdx.x == 0) { fb_row[r] = 1; atomicExch(fb_any, 1); }
        return;
    }
    for (int i = threadIdx.x; i < nwords; i += TopkCfg<T>::kThreads) tie[i] = 0u;
    uint32_t need;
    const uint32_t tau = slice_radix_select<T>(sh, (uint32_t)k, true, &need);
    {
        const int lo = warp * TopkCfg<T>::kSlice, cnt = (int)sh.wcount[warp];
        for (int i = lane; i < cnt; i += 32) {
            const uint32_t key = sh.cand_key[lo + i];
            const int s = sh.cand_idx[lo + i];
            if (key > tau) atomicOr(&sel[s >> 5], 1u << (s & 31));
            else if (key == tau) atomicOr(&tie[s >> 5], 1u << (s & 31));
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) fb_row[r] = 0;
    trim_ties_and_compact<T>(sh, sel, tie, nwords, need, k, out);
}
}  // namespace

size_t topk_smem_bytes(int max_len) {
    const size_t words = (size_t)(max_len + 31) / 32;
    return sizeof(TopkScratch) + 2 * words * sizeof(uint32_t);
}

int topk_sample_max() { return kSampleMax; }

cudaError_t launch_topk_threshold(const float* sample, long long ld_sample, int q_begin, int rows,
                                  int tile_stride, int k, uint32_t* tau, int* fb_any,
                                  cudaStream_t stream) {
    const int grid = (rows + kRowWarps - 1) / kRowWarps;
    topk_threshold_kernel<<<grid, 32 * kRowWarps, 0, stream>>>(sample, ld_sample, q_begin, rows,
                                                                tile_stride, k, tau, fb_any);
    count_launch(DSA_KERNEL_TOPK);
    return cudaGetLastError();
}

cudaError_t launch_topk_candidates(const uint2* cand, const uint32_t* ccount, int cq,
                                   int nchunk_max, int q_begin, int rows, int max_len, int k,
                                   int* idx, long long ld_idx, int* fb_row, int* fb_any,
                                   cudaStream_t stream) {
    const size_t smem = topk_smem_bytes(max_len);
    cudaError_t e = cudaFuncSetAttribute(topk_candidates_kernel<512>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_candidates_kernel<512><<<rows, 512, smem, stream>>>(cand, ccount, cq, nchunk_max,
                                                             q_begin, max_len, k, idx, ld_idx,
                                                             fb_row, fb_any);
    count_launch(DSA_KERNEL_TOPK);
    return cudaGetLastError();
}

}  // namespace dsa
