// topk_stream.cu -- per-row top-k of dense fp32 indexer scores: one pass over the row, no
// sort, no per-key bitmap.
//
// Selection rule (DSA ablation card, "Attention" bullet and closing note): the k largest
// of the row's n valid scores, equal scores resolved towards the lower key index; if
// n <= k every key is selected.  Output: the selected key positions in ascending order,
// then -1 padding.
//
// One small CTA per row (256 threads, about 36 KB of shared memory at 65536 keys, so four
// rows are in flight on every SM), longest rows first.  A launch with fewer rows than the
// GPU has SMs gives each row 1024 threads, or, with at most half as many rows as SMs, a
// cluster of two 512-thread CTAs that split the stream phase and gather the candidates in
// the first CTA's buffer through distributed shared memory.
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
// the row for tau and need, then one ordered pass with a block scan per four keys of every
// thread.
#include <cooperative_groups.h>

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

// Valid length of row r (-1: a row the caller did not ask for).
__device__ __forceinline__ int row_length(int r, int q_begin, const int* __restrict__ row_len,
                                          int max_len, const int* __restrict__ row_mask,
                                          unsigned* __restrict__ err) {
    if (row_mask != nullptr && row_mask[r] == 0) return -1;
    if (row_len == nullptr) return q_begin + r + 1;
    const int n = row_len[r];
    if (n < 0 || n > max_len) {
        if (threadIdx.x == 0) atomicOr(err, DSA_DEVERR_INDEX_RANGE);
        return n < 0 ? 0 : max_len;
    }
    return n;
}

// Sample phase (rows longer than the candidate buffer): the provisional threshold tau0, the
// lower edge of the 16-bit bin that holds the sample key of rank e + 4 sqrt(e) + 2.
template <int NT>
__device__ __forceinline__ uint32_t sample_threshold(const float* __restrict__ row, int n, int k,
                                                     StreamSmem& sm) {
    using C = SCfg<NT>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
    return block_radix_select<NT, C::kSPT>(sk, rank, fixed, hi, 16, sm, &unused) & 0xFFFF0000u;
}

// Stream phase over chunks [cb, ce) of the row: every score >= tau0f goes to sm.cand,
// appended at sm.ncand (which may pass kCap: entries past it are not stored), and each chunk
// records where its candidates start and how many there are.  Positions past the row or
// past chunk ce read as NaN, which no comparison takes.
template <int NT>
__device__ __forceinline__ void stream_candidates(const float* __restrict__ row, int n,
                                                  float tau0f, int cb, int ce,
                                                  uint16_t* chunk_start, uint8_t* chunk_cnt,
                                                  StreamSmem& sm) {
    using C = SCfg<NT>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nend = min(n, ce * kChunk);
    const int nfull = nend / kChunk;  // chunks that lie entirely inside [0, nend)
    for (int c0 = cb + warp; c0 < ce; c0 += C::kWarps * C::kUnroll) {
        float4 v[C::kUnroll];
#pragma unroll
        for (int u = 0; u < C::kUnroll; ++u) {
            const int c = c0 + u * C::kWarps;
            const int s0 = c * kChunk + 4 * lane;
            if (c < nfull) {
                v[u] = __ldcs(reinterpret_cast<const float4*>(row + s0));
            } else {
                v[u].x = s0 < nend ? __ldcs(row + s0) : __int_as_float(0x7fc00000);
                v[u].y = s0 + 1 < nend ? __ldcs(row + s0 + 1) : __int_as_float(0x7fc00000);
                v[u].z = s0 + 2 < nend ? __ldcs(row + s0 + 2) : __int_as_float(0x7fc00000);
                v[u].w = s0 + 3 < nend ? __ldcs(row + s0 + 3) : __int_as_float(0x7fc00000);
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
            if (c < ce) {
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
}

// Select and output phases over the ncand (k <= ncand <= kCap) candidates of chunks
// [0, nch): tau = the k-th largest candidate, need = the selected keys equal to tau, then
// every selected key's position written to out in ascending order.
template <int NT>
__device__ __forceinline__ void select_and_output(uint32_t ncand, int nch, int k,
                                                  const uint16_t* chunk_start,
                                                  const uint8_t* chunk_cnt, int* out,
                                                  int idx_offset, StreamSmem& sm) {
    using C = SCfg<NT>;
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

    // threads take consecutive chunks; one scan places every selected key (scores are
    // compared as floats with tau's own value: x > tauf exactly when float_order_key(x) >
    // tau, and x == tauf when the keys are equal, -0 == +0 included)
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

// One CTA per row.
template <int NT>
__global__ void __launch_bounds__(NT, NT >= 1024 ? 1 : 4)
topk_stream_kernel(const float* __restrict__ scores, long long ld, int rows, int q_begin,
                   const int* __restrict__ row_len, int max_len, int k, int* __restrict__ idx,
                   long long ld_idx, const int* __restrict__ row_mask, int idx_offset,
                   unsigned* __restrict__ err) {
    chained_launch_gate();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StreamSmem& sm = *reinterpret_cast<StreamSmem*>(smem_raw);
    const int max_chunks = (max_len + kChunk - 1) / kChunk;
    uint16_t* chunk_start = reinterpret_cast<uint16_t*>(smem_raw + sizeof(StreamSmem));
    uint8_t* chunk_cnt = reinterpret_cast<uint8_t*>(chunk_start + max_chunks);

    // causal rows grow with r: the longest rows go first so that the launch ends on short
    // ones
    const int r = row_len != nullptr ? (int)blockIdx.x : rows - 1 - (int)blockIdx.x;
    const int n = row_length(r, q_begin, row_len, max_len, row_mask, err);
    if (n < 0) return;
    int* out = idx + (long long)r * ld_idx;
    if (n <= k) {  // every valid key is selected
        for (int i = threadIdx.x; i < k; i += NT) out[i] = i < n ? i + idx_offset : -1;
        return;
    }
    const float* row = scores + (long long)r * ld;
    if (threadIdx.x == 0) sm.ncand = 0u;
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[0][i] = 0u;

    const uint32_t tau0 = n > kCap ? sample_threshold<NT>(row, n, k, sm) : 0u;
    // x >= tau0f exactly when float_order_key(x) >= tau0 (for tau0 = 0: every score);
    // positions past the row read as NaN, which no comparison takes
    const float tau0f = tau0 == 0u ? -INFINITY : order_key_to_float(tau0);
    const int nch = (n + kChunk - 1) / kChunk;
    stream_candidates<NT>(row, n, tau0f, 0, nch, chunk_start, chunk_cnt, sm);
    __syncthreads();
    const uint32_t ncand = sm.ncand;
    if (ncand < (uint32_t)k || ncand > (uint32_t)kCap) {  // block-uniform
        exact_from_global<NT>(row, n, k, out, idx_offset, sm);
        return;
    }
    select_and_output<NT>(ncand, nch, k, chunk_start, chunk_cnt, out, idx_offset, sm);
}

// A cluster of CTAs per row, for launches with few rows (a decode batch).  Every CTA computes the same tau0 from the same sample and streams its own range
// of chunks into its own candidate buffer; the candidate counts are read across the
// cluster through distributed shared memory, every CTA copies its candidates and chunk
// records into CTA 0's buffer behind those of the CTAs before it (the row order), and CTA
// 0 selects and writes the row.  Two cluster barriers: after the stream (the counts are
// final) and after the copies (they are visible to CTA 0, and no CTA reads another's
// shared memory after it, so the others may exit).
template <int NT>
__global__ void __launch_bounds__(NT, 1024 / NT)
topk_cluster_kernel(const float* __restrict__ scores, long long ld, int rows, int q_begin,
                    const int* __restrict__ row_len, int max_len, int k, int* __restrict__ idx,
                    long long ld_idx, const int* __restrict__ row_mask, int idx_offset,
                    unsigned* __restrict__ err) {
    namespace cg = cooperative_groups;
    chained_launch_gate();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StreamSmem& sm = *reinterpret_cast<StreamSmem*>(smem_raw);
    const int max_chunks = (max_len + kChunk - 1) / kChunk;
    uint16_t* chunk_start = reinterpret_cast<uint16_t*>(smem_raw + sizeof(StreamSmem));
    uint8_t* chunk_cnt = reinterpret_cast<uint8_t*>(chunk_start + max_chunks);
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned crank = cluster.block_rank(), csize = cluster.num_blocks();

    // every CTA of a cluster takes the same row, so each return below is cluster-uniform
    const int rid = (int)(blockIdx.x / csize);
    const int r = row_len != nullptr ? rid : rows - 1 - rid;
    const int n = row_length(r, q_begin, row_len, max_len, row_mask, err);
    if (n < 0) return;
    int* out = idx + (long long)r * ld_idx;
    if (n <= k) {
        if (crank == 0)
            for (int i = threadIdx.x; i < k; i += NT) out[i] = i < n ? i + idx_offset : -1;
        return;
    }
    const float* row = scores + (long long)r * ld;
    if (threadIdx.x == 0) sm.ncand = 0u;
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[0][i] = 0u;

    const uint32_t tau0 = n > kCap ? sample_threshold<NT>(row, n, k, sm) : 0u;
    const float tau0f = tau0 == 0u ? -INFINITY : order_key_to_float(tau0);
    const int nch = (n + kChunk - 1) / kChunk;
    const int per = (nch + (int)csize - 1) / (int)csize;
    const int cb = min((int)crank * per, nch), ce = min(cb + per, nch);
    stream_candidates<NT>(row, n, tau0f, cb, ce, chunk_start, chunk_cnt, sm);
    __syncthreads();
    cluster.sync();  // every CTA's count is final

    uint32_t before = 0, total = 0;
    for (unsigned j = 0; j < csize; ++j) {
        const uint32_t c = *cluster.map_shared_rank(&sm.ncand, j);
        before += j < crank ? c : 0u;
        total += c;
    }
    const bool exact = total < (uint32_t)k || total > (uint32_t)kCap;  // cluster-uniform
    if (!exact && crank != 0) {
        // total <= kCap: every CTA stored all of its candidates
        const uint32_t mine = sm.ncand;
        uint2* dst = cluster.map_shared_rank(sm.cand, 0);
        for (uint32_t i = threadIdx.x; i < mine; i += NT) dst[before + i] = sm.cand[i];
        uint16_t* dst_start = cluster.map_shared_rank(chunk_start, 0);
        uint8_t* dst_cnt = cluster.map_shared_rank(chunk_cnt, 0);
        for (int c = cb + (int)threadIdx.x; c < ce; c += NT) {
            dst_start[c] = (uint16_t)(chunk_start[c] + before);
            dst_cnt[c] = chunk_cnt[c];
        }
    }
    cluster.sync();  // the copies are visible to CTA 0; no remote access follows
    if (crank != 0) return;
    if (exact) {
        exact_from_global<NT>(row, n, k, out, idx_offset, sm);
        return;
    }
    select_and_output<NT>(total, nch, k, chunk_start, chunk_cnt, out, idx_offset, sm);
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
    if (rows >= ctx.num_sms) {
        auto kernel = topk_stream_kernel<256>;
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_chained(kernel, dim3(rows), dim3(256), smem, stream, 1, scores, ld, rows, q_begin,
                           row_len, max_len, k, idx, ld_idx, row_mask, idx_offset, ctx.err);
        count_launch(DSA_KERNEL_TOPK);
        return e;
    }
    // At most half as many rows as SMs (a decode batch): a pair of 512-thread CTAs per row
    // (a cluster of two), which halves the candidate pass of each row and keeps the
    // row-level phases on 512 threads.  Measured on 64 rows of 32768 keys: 14.5 us against
    // 15.7 us for one 1024-thread CTA per row; clusters of four or eight 256- or 512-thread
    // CTAs were slower (16.3 to 26.4 us), their row-level phases running on fewer threads.
    const int max_chunks = (max_len + kChunk - 1) / kChunk;
    constexpr int kClusterThreads = 512, cl = 2;
    if (2 * rows <= ctx.num_sms && max_chunks >= 32) {
        auto kernel = topk_cluster_kernel<kClusterThreads>;
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_chained(kernel, dim3((unsigned)(rows * cl)), dim3(kClusterThreads), smem, stream,
                           (unsigned)cl, scores, ld, rows, q_begin, row_len, max_len, k, idx,
                           ld_idx, row_mask, idx_offset, ctx.err);
        count_launch(DSA_KERNEL_TOPK);
        return e;
    }
    auto kernel = topk_stream_kernel<1024>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_chained(kernel, dim3(rows), dim3(1024), smem, stream, 1, scores, ld, rows, q_begin,
                       row_len, max_len, k, idx, ld_idx, row_mask, idx_offset, ctx.err);
    count_launch(DSA_KERNEL_TOPK);
    return e;
}

}  // namespace dsa

