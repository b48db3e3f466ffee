// topk_stream.cu -- per-row top-k of dense fp32 indexer scores: one pass over the row, no
// sort, no per-key bitmap.
//
// Selection rule (DSA ablation card, "Attention" bullet and closing note): the k largest
// of the row's n valid scores, equal scores resolved towards the lower key index; if
// n <= k every key is selected.  Output: the selected key positions in ascending order,
// then -1 padding.
//
// One small CTA per row (256 threads, about 36 KB of shared memory at 65536 keys, so four
// rows are in flight on every SM; 1024 threads when a launch has fewer rows than the GPU
// has SMs), longest rows first.
// Scores map to order-preserving uint32 keys (-0 like +0).
//   sample  rows longer than the candidate buffer load up to 4096 scores (32-key pieces
//           spread evenly over the row) into registers; radix selection (8-bit digits,
//           below the bits the sample's smallest and largest keys share) gives the top
//           16 bits of the sample key of rank e + 4 sqrt(e) + 2, e = the number of samples
//           expected above the row's k-th largest score; the lower edge tau0 of that
//           16-bit bin is the provisional threshold;
//   stream  one pass over the row, 128-key chunks (one 16-byte load per lane), four per
//           warp and iteration, dealt to the warps round-robin: every score >= tau0 goes to
//           the candidate buffer as {score bits, position in the chunk}, the chunk's candidates
//           contiguous and in index order.  Each lane's 4-bit take mask per chunk and the
//           counts packed one byte per chunk give, after one warp scan, every candidate its
//           place in a range reserved with one shared atomic per warp and iteration; each
//           chunk records where its candidates start and how many there are;
//   select  the candidates' keys move to registers; radix selection with 8-bit digits
//           (a shared histogram per digit, two barriers) below the bits that the smallest
//           and largest candidate share gives the k-th largest key tau and `need`, the
//           number of keys equal to tau that are selected;
//   output  threads take consecutive chunks, count their selected keys and ties, and one
//           block-wide exclusive scan (both counts packed in one word) gives every
//           selected key its output position: ascending order without sorting.
// Rows whose candidates number fewer than k or more than the buffer holds (a sample that
// misled, heavy ties) are redone exactly from global memory: four 8-bit radix passes over
// the row for tau and need, then one ordered pass with a block scan per 1024 keys.
#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

constexpr int kChunk = 128;        // keys per chunk: one float4 per lane of a warp
constexpr int kCap = 4096;         // candidate buffer entries
constexpr int kSamples = 4096;     // sampled keys at most

template <int NT>
struct SCfg {
    static constexpr int kWarps = NT / 32;
    static constexpr int kCPT = kCap / NT;       // candidates per thread in the select
    static constexpr int kSPT = kSamples / NT;   // samples per thread
    static constexpr int kUnroll = NT >= 1024 ? 2 : 4;  // chunks in flight per warp
    static_assert(kCap % NT == 0 && kSamples % NT == 0 && kSamples % 32 == 0, "block size");
};

struct StreamSmem {
    uint2 cand[kCap];             // candidates: {score bits, position within the chunk}
    uint32_t hist[2][256];        // radix histograms, alternating between rounds
    uint32_t red[32][2];          // per-warp partials of a reduction
    uint32_t scan[32];
    uint32_t ncand;               // candidates appended (may exceed kCap)
    uint32_t bcast[2];
    // followed by chunk_start[nchunk] (uint16) and chunk_cnt[nchunk] (uint8)
};

// The float threshold equivalent to an order key: float_order_key(x) >= key0 exactly when
// x >= key_to_float_lower(key0), for key0 != 0 and x not NaN.
__device__ __forceinline__ float order_key_to_float(uint32_t key0) {
    return __uint_as_float((key0 & 0x80000000u) ? (key0 & 0x7FFFFFFFu) : ~key0);
}

// Bits pos .. pos + len - 1 of v (PTX bfe: one instruction).
__device__ __forceinline__ uint32_t bfe_u32(uint32_t v, int pos, int len) {
    uint32_t r;
    asm("bfe.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(pos), "r"(len));
    return r;
}

// Block-wide minimum and maximum of the keys that are not 0 (0 marks an absent entry).
template <int NT, int N>
__device__ __forceinline__ void block_minmax(const uint32_t (&keys)[N], uint32_t* mn_out,
                                             uint32_t* mx_out, StreamSmem& sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        mn = min(mn, keys[i] ? keys[i] : 0xFFFFFFFFu);
        mx = max(mx, keys[i]);
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) {
        sm.red[warp][0] = mn;
        sm.red[warp][1] = mx;
    }
    __syncthreads();
    mn = __reduce_min_sync(0xffffffffu, lane < SCfg<NT>::kWarps ? sm.red[lane][0] : 0xFFFFFFFFu);
    mx = __reduce_max_sync(0xffffffffu, lane < SCfg<NT>::kWarps ? sm.red[lane][1] : 0u);
    *mn_out = mn;
    *mx_out = mx;
}

// Warp 0: the digit D (from the top of a 256-bin histogram) with
// above(D) < rank <= above(D) + hist[D], above(D) = the count in bins above D; D and
// above(D) go to sm.bcast.
__device__ __forceinline__ void find_digit_from_top(const uint32_t* hist, uint32_t rank,
                                                    StreamSmem& sm) {
    const int lane = threadIdx.x & 31;
    uint32_t c[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * lane - i];
        local += c[i];
    }
    uint32_t x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    uint32_t above = x - local;
    if (above < rank && above + local >= rank) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (above < rank && above + c[i] >= rank) {
                sm.bcast[0] = (uint32_t)(255 - 8 * lane - i);
                sm.bcast[1] = above;
            }
            above += c[i];
        }
    }
}

// Radix selection with 8-bit digits among the block's keys (0 = absent entry).  Every key
// present has the bits >= hi of `prefix`; sm.hist[0] is zero on entry (behind a barrier).
// Returns the rank-th largest key with its bits < lo cleared, and sets *rank_out to rank
// minus the number of keys above that truncated value's bin: for lo = 0, how many of the
// keys equal to the result belong to the top `rank`.  Two barriers per digit: the next
// round's histogram is cleared while this one fills.
template <int NT, int N>
__device__ uint32_t block_radix_select(const uint32_t (&keys)[N], uint32_t rank, uint32_t prefix,
                                       int hi, int lo, StreamSmem& sm, uint32_t* rank_out) {
    const int warp = threadIdx.x >> 5;
    int b = hi, h = 0;
    while (b > lo) {
        const int d = min(8, b - lo);
        const int s = b - d;
        uint32_t* hist = sm.hist[h];
        for (int i = threadIdx.x; i < 256; i += NT) sm.hist[h ^ 1][i] = 0u;
        const uint32_t hp = b >= 32 ? 0u : prefix >> b;
        if (b < 32 && hp != 0u) {
            // an absent entry (key 0) cannot match a non-zero prefix: no test for it
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const uint32_t key = keys[i];
                if ((key >> b) == hp) atomicAdd(&hist[bfe_u32(key, s, d)], 1u);
            }
        } else {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const uint32_t key = keys[i];
                if (key != 0u && (b >= 32 || (key >> b) == hp)) atomicAdd(&hist[bfe_u32(key, s, d)], 1u);
            }
        }
        __syncthreads();
        if (warp == 0) find_digit_from_top(hist, rank, sm);
        __syncthreads();
        prefix |= sm.bcast[0] << s;
        rank -= sm.bcast[1];
        b = s;
        h ^= 1;
    }
    if (h) {  // leave sm.hist[0] zero for the next caller
        __syncthreads();
        for (int i = threadIdx.x; i < 256; i += NT) sm.hist[0][i] = 0u;
        __syncthreads();
    }
    *rank_out = rank;
    return prefix;
}

// Exclusive prefix sum over the block's threads in thread order; *total gets the sum.
template <int NT>
__device__ __forceinline__ uint32_t block_scan_excl(uint32_t v, StreamSmem& sm, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm.scan[warp] = x;
    __syncthreads();
    uint32_t before = x - v, tot = 0;
#pragma unroll
    for (int w = 0; w < SCfg<NT>::kWarps; ++w) {
        const uint32_t s = sm.scan[w];
        before += w < warp ? s : 0u;
        tot += s;
    }
    __syncthreads();  // sm.scan may be rewritten by the next scan
    *total = tot;
    return before;
}

// Adds 1 to hist[bin] for every lane with pred, one shared atomic per distinct bin.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool pred) {
    const unsigned active = __ballot_sync(0xffffffffu, pred);
    if (pred) {
        const unsigned peers = __match_any_sync(active, bin);
        if ((int)lane_id() == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
}

// Loads the 4 scores of chunk position s0..s0+3 (zero past n).
__device__ __forceinline__ float4 load4(const float* __restrict__ row, int s0, int n) {
    if (s0 + 3 < n) return __ldcs(reinterpret_cast<const float4*>(row + s0));
    float4 v;
    v.x = s0 < n ? __ldcs(row + s0) : 0.f;
    v.y = s0 + 1 < n ? __ldcs(row + s0 + 1) : 0.f;
    v.z = s0 + 2 < n ? __ldcs(row + s0 + 2) : 0.f;
    v.w = 0.f;
    return v;
}

// Exact selection from global memory (rows the candidate buffer cannot settle): tau and
// need by four 8-bit radix passes over the row, then the selected positions in index
// order, 4 keys per thread and one block scan per NT * 4 keys.
template <int NT>
__device__ void exact_from_global(const float* __restrict__ row, int n, int k, int* out,
                                  int idx_offset, StreamSmem& sm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t* hist = sm.hist[1];
    uint32_t prefix = 0u, rank = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0u;
        __syncthreads();
        for (int base = warp * kChunk; base < n; base += SCfg<NT>::kWarps * kChunk) {
            const int s0 = base + 4 * lane;
            const float4 v = load4(row, s0, n);
            const float xv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t key = float_order_key(xv[e]);
                const bool in = s0 + e < n &&
                                (pass == 0 || (key >> (shift + 8)) == (prefix >> (shift + 8)));
                hist_add(hist, (key >> shift) & 0xFFu, in);
            }
        }
        __syncthreads();
        if (warp == 0) find_digit_from_top(hist, rank, sm);
        __syncthreads();
        prefix |= sm.bcast[0] << shift;
        rank -= sm.bcast[1];
        __syncthreads();
    }
    const uint32_t tau = prefix, need = rank;
    uint32_t sel_run = 0, tie_run = 0;
    for (int base = 0; base < n; base += NT * 4) {
        const int s0 = base + 4 * threadIdx.x;
        const float4 v = load4(row, s0, n);
        const float xv[4] = {v.x, v.y, v.z, v.w};
        uint32_t key[4], packed = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            key[e] = float_order_key(xv[e]);
            const bool in = s0 + e < n;
            packed += (in && key[e] > tau) ? 1u : 0u;
            packed += (in && key[e] == tau) ? 0x10000u : 0u;
        }
        uint32_t total;
        const uint32_t before = block_scan_excl<NT>(packed, sm, &total);
        uint32_t sb = sel_run + (before & 0xFFFFu), tb = tie_run + (before >> 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (s0 + e >= n) continue;
            if (key[e] > tau) {
                out[sb + min(tb, need)] = s0 + e + idx_offset;
                ++sb;
            } else if (key[e] == tau) {
                if (tb < need) out[sb + tb] = s0 + e + idx_offset;
                ++tb;
            }
        }
        sel_run += total & 0xFFFFu;
        tie_run += total >> 16;
    }
}

template <int NT>
__global__ void __launch_bounds__(NT, NT >= 1024 ? 1 : 4)
topk_stream_kernel(const float* __restrict__ scores, long long ld, int rows, int q_begin,
                   const int* __restrict__ row_len, int max_len, int k, int* __restrict__ idx,
                   long long ld_idx, const int* __restrict__ row_mask, int idx_offset,
                   unsigned* __restrict__ err) {
    using C = SCfg<NT>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StreamSmem& sm = *reinterpret_cast<StreamSmem*>(smem_raw);
    const int max_chunks = (max_len + kChunk - 1) / kChunk;
    uint16_t* chunk_start = reinterpret_cast<uint16_t*>(smem_raw + sizeof(StreamSmem));
    uint8_t* chunk_cnt = reinterpret_cast<uint8_t*>(chunk_start + max_chunks);

    // causal rows grow with r: the longest rows go first so that the launch ends on short
    // ones
    const int r = row_len != nullptr ? (int)blockIdx.x : rows - 1 - (int)blockIdx.x;
    if (row_mask != nullptr && row_mask[r] == 0) return;  // row not asked for
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int n;
    if (row_len != nullptr) {
        n = row_len[r];
        if (n < 0 || n > max_len) {
            if (threadIdx.x == 0) atomicOr(err, DSA_DEVERR_INDEX_RANGE);
            n = n < 0 ? 0 : max_len;
        }
    } else {
        n = q_begin + r + 1;
    }
    int* out = idx + (long long)r * ld_idx;
    if (n <= k) {  // every valid key is selected
        for (int i = threadIdx.x; i < k; i += NT) out[i] = i < n ? i + idx_offset : -1;
        return;
    }
    const float* row = scores + (long long)r * ld;
    if (threadIdx.x == 0) sm.ncand = 0u;
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[0][i] = 0u;

    // ---- provisional threshold tau0 from a sample (rows longer than the buffer) ----
    uint32_t tau0 = 0u;
    if (n > kCap) {
        const int nch32 = (n + 31) >> 5;
        const int stride = (nch32 + kSamples / 32 - 1) / (kSamples / 32);
        const int nsc = (nch32 + stride - 1) / stride;  // sampled 32-key pieces
        uint32_t sk[C::kSPT];
#pragma unroll
        for (int i = 0; i < C::kSPT; ++i) {
            const int j = warp + i * C::kWarps;
            const int s = j * stride * 32 + lane;
            sk[i] = (j < nsc && s < n) ? float_order_key(__ldg(row + s)) : 0u;
        }
        const int last0 = (nsc - 1) * stride * 32;
        const int m = (nsc - 1) * 32 + min(32, n - last0);
        const float e = (float)k * (float)m / (float)n;
        uint32_t rank = (uint32_t)ceilf(e + 4.f * sqrtf(e)) + 2u;
        if (rank > (uint32_t)m) rank = (uint32_t)m;
        uint32_t mn, mx, unused;
        block_minmax<NT, C::kSPT>(sk, &mn, &mx, sm);
        const uint32_t diff = mn ^ mx;
        const int hi = diff ? 32 - __clz(diff) : 0;
        const uint32_t fixed = hi >= 32 ? 0u : (mx & ~((1u << hi) - 1u));
        tau0 = block_radix_select<NT, C::kSPT>(sk, rank, fixed, hi, 16, sm, &unused) & 0xFFFF0000u;
    }
    // x >= tau0f exactly when float_order_key(x) >= tau0 (for tau0 = 0: every score);
    // positions past the row read as NaN, which no comparison takes
    const float tau0f = tau0 == 0u ? -INFINITY : order_key_to_float(tau0);

    // ---- stream: every key >= tau0 to the candidate buffer, chunk by chunk ----
    const int nch = (n + kChunk - 1) / kChunk;
    const int nfull = n / kChunk;  // chunks that lie entirely inside the row
    for (int c0 = warp; c0 < nch; c0 += C::kWarps * C::kUnroll) {
        float4 v[C::kUnroll];
#pragma unroll
        for (int u = 0; u < C::kUnroll; ++u) {
            const int c = c0 + u * C::kWarps;
            const int s0 = c * kChunk + 4 * lane;
            if (c < nfull) {
                v[u] = __ldcs(reinterpret_cast<const float4*>(row + s0));
            } else {
                v[u].x = s0 < n ? __ldcs(row + s0) : __int_as_float(0x7fc00000);
                v[u].y = s0 + 1 < n ? __ldcs(row + s0 + 1) : __int_as_float(0x7fc00000);
                v[u].z = s0 + 2 < n ? __ldcs(row + s0 + 2) : __int_as_float(0x7fc00000);
                v[u].w = s0 + 3 < n ? __ldcs(row + s0 + 3) : __int_as_float(0x7fc00000);
            }
        }
        // per lane: the 4-bit take mask of each unrolled chunk, and the counts packed one
        // byte per chunk (at most 4 per lane, 128 per chunk: no byte overflows), so that
        // one warp scan places the candidates of all of them
        uint32_t msk[C::kUnroll], packed = 0;
#pragma unroll
        for (int u = 0; u < C::kUnroll; ++u) {
            msk[u] = (v[u].x >= tau0f ? 1u : 0u) | (v[u].y >= tau0f ? 2u : 0u) |
                     (v[u].z >= tau0f ? 4u : 0u) | (v[u].w >= tau0f ? 8u : 0u);
            packed |= (uint32_t)__popc(msk[u]) << (8 * u);
        }
        uint32_t incl = packed;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t chunk_tot = __shfl_sync(0xffffffffu, incl, 31);  // per-chunk totals
        const uint32_t excl = incl - packed;
        uint32_t tot = 0;
#pragma unroll
        for (int u = 0; u < C::kUnroll; ++u) tot += (chunk_tot >> (8 * u)) & 0xFFu;
        uint32_t base = 0;
        if (lane == 0 && tot) base = atomicAdd(&sm.ncand, tot);
        base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
        for (int u = 0; u < C::kUnroll; ++u) {
            const int c = c0 + u * C::kWarps;
            const uint32_t cnt = (chunk_tot >> (8 * u)) & 0xFFu;
            if (c < nch) {
                if (lane == 0) {
                    chunk_start[c] = (uint16_t)min(base, 0xFFFFu);
                    chunk_cnt[c] = (uint8_t)cnt;
                }
                // a chunk past the buffer's end sends the row to the exact path
                if (base + cnt <= (uint32_t)kCap) {
                    uint32_t pos = base + ((excl >> (8 * u)) & 0xFFu);
                    const float xv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if ((msk[u] >> e) & 1u) {
                            sm.cand[pos] = make_uint2(__float_as_uint(xv[e]), (uint32_t)(4 * lane + e));
                            ++pos;
                        }
                    }
                }
            }
            base += cnt;
        }
    }
    __syncthreads();
    const uint32_t ncand = sm.ncand;
    if (ncand < (uint32_t)k || ncand > (uint32_t)kCap) {  // block-uniform
        exact_from_global<NT>(row, n, k, out, idx_offset, sm);
        return;
    }

    // ---- select: tau = k-th largest candidate, need = selected keys equal to tau ----
    uint32_t ck[C::kCPT];
#pragma unroll
    for (int i = 0; i < C::kCPT; ++i) {
        const uint32_t j = threadIdx.x + i * NT;
        ck[i] = j < ncand ? float_order_key(__uint_as_float(sm.cand[j].x)) : 0u;
    }
    uint32_t mn, mx, need;
    block_minmax<NT, C::kCPT>(ck, &mn, &mx, sm);
    // every candidate lies in [mn, mx]: the bits above their highest difference are fixed
    const uint32_t diff = mn ^ mx;
    const int hi = diff ? 32 - __clz(diff) : 0;
    const uint32_t fixed = hi >= 32 ? 0u : (mx & ~((1u << hi) - 1u));
    const uint32_t tau = block_radix_select<NT, C::kCPT>(ck, (uint32_t)k, fixed, hi, 0, sm, &need);

    // ---- output: threads take consecutive chunks; one scan places every selected key ----
    // (scores are compared as floats with tau's own value: x > tauf exactly when
    // float_order_key(x) > tau, and x == tauf when the keys are equal, -0 == +0 included)
    const float tauf = order_key_to_float(tau);
    const int cpt = (nch + NT - 1) / NT;
    const int ca = min((int)threadIdx.x * cpt, nch), cb = min(ca + cpt, nch);
    uint32_t packed = 0;
    for (int c = ca; c < cb; ++c) {
        const int st = chunk_start[c], ct = chunk_cnt[c];
        for (int j = st; j < st + ct; ++j) {
            const float x = __uint_as_float(sm.cand[j].x);
            packed += x > tauf ? 1u : (x == tauf ? 0x10000u : 0u);
        }
    }
    uint32_t total;
    const uint32_t before = block_scan_excl<NT>(packed, sm, &total);
    uint32_t sb = before & 0xFFFFu, tb = before >> 16;
    for (int c = ca; c < cb; ++c) {
        const int st = chunk_start[c], ct = chunk_cnt[c];
        for (int j = st; j < st + ct; ++j) {
            const uint2 cj = sm.cand[j];
            const float x = __uint_as_float(cj.x);
            const int s = c * kChunk + (int)cj.y + idx_offset;
            if (x > tauf) {
                out[sb + min(tb, need)] = s;
                ++sb;
            } else if (x == tauf) {
                if (tb < need) out[sb + tb] = s;
                ++tb;
            }
        }
    }
}

}  // namespace

size_t topk_stream_smem_bytes(int max_len) {
    const size_t chunks = (size_t)(max_len + kChunk - 1) / kChunk;
    return sizeof(StreamSmem) + chunks * 3 + 16;
}

cudaError_t launch_topk(const float* scores, long long ld, int rows, int q_begin,
                        const int* row_len, int max_len, int k, int* idx, long long ld_idx,
                        cudaStream_t stream, const DevCtx& ctx, const int* row_mask,
                        int idx_offset) {
    const size_t smem = topk_stream_smem_bytes(max_len);
    // fewer rows than SMs (a decode batch): 1024 threads per row shorten each row's chain
    const bool wide = rows < ctx.num_sms;
    auto kernel = wide ? topk_stream_kernel<1024> : topk_stream_kernel<256>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<rows, wide ? 1024 : 256, smem, stream>>>(scores, ld, rows, q_begin, row_len, max_len,
                                                      k, idx, ld_idx, row_mask, idx_offset,
                                                      ctx.err);
    count_launch(DSA_KERNEL_TOPK);
    return cudaGetLastError();
}

}  // namespace dsa

