// Steps 3-5 of AB-Sparse (arXiv 2605.12110), Fig. 1: query-centroid dot
// product estimation over INT4 centroid codes, per-head top-K block
// selection under a token budget (Fig. 9), and exact softmax attention over
// the selected blocks' tokens gathered from the paged cache.
//
// One thread-block cluster of C CTAs (C in 1..16) handles one
// (sequence, KV head).  Phases of decode_kernel:
//   A  score:   CTA r streams its contiguous 1/C share of the head's code
//               rows into shared memory with 1-D bulk copies through a ring
//               of 16 KB stages, scores every row (8 lanes per 64-byte row,
//               16 codes per lane, 4 rows per lane group at once, codes fed
//               to packed f32x2 FMAs as exact subnormals, fp32 sums) and
//               sends each group of 4 scores to the other CTAs of the
//               cluster with asynchronous 16-byte distributed-shared-memory
//               stores that count down the receiver's mbarrier (its own
//               scores with plain stores).  Meanwhile the sequence's
//               page-table row is staged in shared memory (or its entries
//               for the CTA's own rows, when the row does not fit).
//   B  each CTA waits on its own mbarrier until all n_h scores arrived.
//   C  select:  every CTA runs the same deterministic top-K (largest scores,
//               ties to the lower block index): a 1024-bin histogram over the
//               score range finds the bin holding the K-th score, a bitmap
//               marks the scores above it, the few scores in that bin are
//               ranked exactly, and each warp writes its bitmap words'
//               entries of the ascending block list.  A 4 x 8-bit
//               radix select over order-preserving keys covers degenerate
//               ranges.  All CTAs hold the same list without another
//               exchange.
//   D  attend:  the selected blocks expand to bs/16 pages each; CTA r takes a
//               contiguous 1/C share of those pages.  Each warp owns every
//               8th page: it loads the (page, head) K and V slices with 2-D
//               tensor copies (128-byte swizzle, each CTA's own) on its own
//               mbarrier into one of its one or two page buffers (two in the
//               one-CTA-per-SM instance), then computes S^T = Q K^T and O += P V on mma.sync
//               bf16 tiles with the GQA group as the 16-row M dimension and an
//               online softmax in fp32; each warp also bulk-prefetches its
//               next two pages into L2.
//   E  merge:   warps merge in shared memory into the CTA's partial; CTA r
//               owns output channels [r*128/C, (r+1)*128/C) and receives
//               that slice of every CTA's partial (its own included) and
//               every CTA's (m, l) by asynchronous distributed-shared-memory
//               stores counted on its mbarrier, then combines them and
//               writes its slice in bf16.
// Modes: select only (writes sel / sel_count), attend only (reads them) and
// full (A-E in one launch, the selection never leaves the chip).  Centroid
// format (INT4 / BF16) and score aggregation (sum / group max) are template
// parameters, so the default kernel carries no code of the other variants
// (its phases run once per launch and their code is fetched every time).
#include <algorithm>
#include <atomic>
#include <cfloat>
#include <mutex>

#include "absp_internal.cuh"

#ifndef ABSP_PAGE_PREFETCH
#define ABSP_PAGE_PREFETCH 2  // pages a warp prefetches into L2 ahead of its TMA copies
#endif

namespace absp {

#ifdef ABSP_PHASE_STAMPS
// Phase stamps, compiled only into the separate profiling build: thread 0 of
// CTAs 0..159 of a fused launch records globaltimer and clock64 at fixed
// points (index k below), in 64 slots taken in launch order.
__device__ unsigned long long g_stamp_t[64 * 160 * 24];
__device__ long long g_stamp_c[64 * 160 * 24];
int g_stamp_launches = 0;
#endif

namespace {

#ifdef ABSP_PHASE_STAMPS
__device__ __forceinline__ void stampk(int slot, int k) {
    if (threadIdx.x == 0 && slot >= 0 && blockIdx.x < 160) {
        const int i = (slot * 160 + blockIdx.x) * 24 + k;
        g_stamp_t[i] = globaltimer_ns();
        g_stamp_c[i] = clock64();
    }
}
#else
__device__ __forceinline__ void stampk(int, int) {}
#endif

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStageRows = 256;                      // code rows per bulk stage
constexpr int kStages = 2;                           // code ring stages, at least
constexpr int kMaxStages = 4;                        // and at most
constexpr int kStageBytes = kStageRows * kRowBytes;  // 16 KiB
constexpr int kPageSmem = 4 * 2048;                  // K lo/hi, V lo/hi halves
constexpr int kBins = 1024;                          // value histogram
constexpr int kMaxCand = 1024;                       // boundary-bin candidates
constexpr int kMaxBitmapWords = (ABSP_MAX_BLOCKS_PER_HEAD + 31) / 32;
constexpr int kSelectScratch = (kBins + 2 * kMaxCand + kMaxBitmapWords) * 4;
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
    KvDesc kv;
    const uint8_t* codes;
    const float* scale;
    const int32_t* zp;
    const __nv_bfloat16* q;
    __nv_bfloat16* out;
    int32_t* sel;
    int32_t* sel_count;
    int32_t kmax;
    int32_t budget;
    int32_t* err;
    float qk_scale_log2;          // log2(e) / sqrt(128)
    uint32_t regA_off;            // byte offsets inside the aligned smem base
    uint32_t small_off;
    uint32_t qs_off;              // the group's queries, after Small
    uint32_t scratch_off;         // select scratch inside region B
    uint32_t wg_off;              // per-head weights inside region B
    int32_t nstages;              // code ring stages (kStages .. kMaxStages)
    uint32_t ring_off;            // code ring inside region B, past the select scratch
    uint32_t ptrow_off;           // staged page-table row, after the list
    int32_t pt_cap;               // entries the staged row holds (0: none)
    int32_t stamp_slot;           // phase-stamp slot (profiling build), else -1
    int32_t npbuf;                // page buffers per warp (1, or 2 when one CTA per SM is enough)
};

// per-head score weights for the group-max variant: [G][8 lanes][20]
// floats (16 used), padded so the 8 lanes of a row read distinct banks
constexpr int kWgStride = 160;

constexpr int kPtStage = 512;    // page-table entries a CTA stages for its own rows

struct Small {                    // fixed-size shared scratch
    int32_t pt[kPtStage];         // page ids of the pages of this CTA's scored rows
    unsigned long long bar_code[kMaxStages];
    unsigned long long bar_page[2 * kWarps];   // [warp][page buffer]
    unsigned long long bar_merge;
    unsigned long long bar_score;
    float2 cmm[16];               // (min, max) of each cluster CTA's scores
    int32_t misc[16];
    float red[2][kWarps];
    alignas(16) float w[kD];      // qbar[ch] * scale[ch] (pre-scaled for INT4 sum scores)
    float kz[8];                  // per lane group: sum_ch w zp, at the group's scale
    float xs[8];                  // per lane group: 2^X
    float zb[kD];                 // 2^23 + zp[ch]
    float zf[kD];                 // zp[ch]
    alignas(16) uint32_t scan[kWarps];
};

// 2^x by the hardware approximation (relative error ~2^-22, far inside
// the bf16 output; -inf gives +0), and a hardware reciprocal.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float fast_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Monotone (non-decreasing) map of a score onto kBins bins of [mn, mx].
// (x - mn) * inv >= 0 for x >= mn; adding 2^23 rounding toward zero puts
// its integer part in the low mantissa bits (an ALU floor, no conversion).
__device__ __forceinline__ int value_bin(float x, float mn, float inv) {
    const float y = fminf((x - mn) * inv, static_cast<float>(kBins - 1));
    return __float_as_int(__fadd_rz(y, 8388608.0f)) - 0x4B000000;
}

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) {
    return *reinterpret_cast<const uint32_t*>(p);
}

// (a0, a1) += (w0, w1) * (r0, r1) as one packed f32x2 FMA, r given as bits.
__device__ __forceinline__ void fma2_bits(float& a0, float& a1, uint32_t r0, uint32_t r1,
                                          float w0, float w1) {
    asm("{\n\t.reg .b64 t, w, c;\n\t"
        "mov.b64 t, {%2, %3};\n\t"
        "mov.b64 w, {%4, %5};\n\t"
        "mov.b64 c, {%0, %1};\n\t"
        "fma.rn.f32x2 c, w, t, c;\n\t"
        "mov.b64 {%0, %1}, c;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "r"(r0), "r"(r1), "f"(w0), "f"(w1));
}

// Dot product of 16 INT4 codes (channel k in nibble k of x.x, then x.y) with
// weights, plus `init`.  Nibble j (0..3) of each 16-bit half is masked in
// place; read as a float, the bits n * 16^j are the subnormal n * 16^j *
// 2^-149, exactly.  w[k] carries the matching 2^(149 - 4j) (times the lane's
// own power-of-two scale), so every product is weight * code times that
// scale, formed exactly as if the code were a float: one AND per channel and
// half a packed FMA, no conversion or unbias step.  Subnormal operands are
// exact and full speed in fma.rn (no .ftz).
__device__ __forceinline__ float int4_dot16(uint2 x, const float (&w)[16], float init) {
    const uint32_t h[4] = {x.x, x.x >> 16, x.y, x.y >> 16};
    float a0 = init, a1 = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        fma2_bits(a0, a1, h[q] & 0xFu, h[q] & 0xF0u, w[4 * q], w[4 * q + 1]);
        fma2_bits(a0, a1, h[q] & 0xF00u, h[q] & 0xF000u, w[4 * q + 2], w[4 * q + 3]);
    }
    return a0 + a1;
}

// Sums of four rows' partial dot products over the 8 lanes of a group
// (lanes 8g .. 8g + 7), returned to every lane of the group.  A transpose
// reduction: each butterfly step halves the rows a lane carries, so lane
// 8g + j ends with the full sum of row j / 2 after three shuffles (instead of
// three per row), then four shuffles gather the rows.
__device__ __forceinline__ float4 group_sum4(const float (&a)[4], int lane) {
    const bool hi = (lane & 4) != 0, mid = (lane & 2) != 0;
    float k0 = hi ? a[2] : a[0], k1 = hi ? a[3] : a[1];
    k0 += __shfl_xor_sync(0xffffffffu, hi ? a[0] : a[2], 4);
    k1 += __shfl_xor_sync(0xffffffffu, hi ? a[1] : a[3], 4);
    float k = mid ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, mid ? k0 : k1, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 1);
    const int base = lane & ~7;
    return make_float4(__shfl_sync(0xffffffffu, k, base), __shfl_sync(0xffffffffu, k, base + 2),
                       __shfl_sync(0xffffffffu, k, base + 4), __shfl_sync(0xffffffffu, k, base + 6));
}

// Block-wide exclusive prefix sum of one uint32 per thread (one barrier;
// `scan` must not be rewritten before the next barrier).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* scan) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) scan[warp] = inc;
    __syncthreads();
    const uint4 a = reinterpret_cast<const uint4*>(scan)[0];
    const uint4 b = reinterpret_cast<const uint4*>(scan)[1];
    const uint32_t t[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t base = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) base += w < warp ? t[w] : 0u;
    return base + inc - v;
}

// Threshold of the top-k by 4 passes of 8-bit radix select over the
// order-preserving keys (keys > T are in, plus `rem` keys equal to T).
__device__ __noinline__ void radix_threshold(const float* sc, int n, int k, uint32_t* hist, Small& sm,
                                uint32_t* T_out, int* rem_out) {
    const int tid = threadIdx.x;
    uint32_t prefix = 0, mask = 0;
    int rem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[tid] = 0;  // kThreads == 256 digits
        __syncthreads();
        for (int i = tid; i < n; i += kThreads) {
            const uint32_t key = order_key(sc[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1u);
        }
        __syncthreads();
        {
            // thread t owns digit 255 - t: an exclusive scan in thread order
            // counts the candidates with a larger digit
            const int dgt = 255 - tid;
            const uint32_t c = hist[dgt];
            const uint32_t above = block_excl_scan(c, sm.scan);
            if (above < static_cast<uint32_t>(rem) && static_cast<uint32_t>(rem) <= above + c) {
                sm.misc[0] = dgt;
                sm.misc[1] = rem - static_cast<int>(above);
            }
        }
        __syncthreads();
        prefix |= static_cast<uint32_t>(sm.misc[0]) << shift;
        mask |= 0xFFu << shift;
        rem = sm.misc[1];
        __syncthreads();
    }
    *T_out = prefix;
    *rem_out = rem;
}

// Ordered compaction of the top-k by a threshold: keys > T are in, and of
// the keys == T the `rem` lowest indices.  Each warp compacts a contiguous
// index range 32 scores at a time with ballots.
__device__ __noinline__ void compact_by_threshold(const float* sc, int n, uint32_t T, int rem,
                                                     int32_t* out, int lo, int hi, Small& sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per_w = (n + kWarps - 1) / kWarps;
    const int w0 = min(n, warp * per_w), w1 = min(n, w0 + per_w);
    uint32_t gt = 0, eq = 0;
    for (int b = w0; b < w1; b += 32) {
        const int i = b + lane;
        const uint32_t key = i < w1 ? order_key(sc[i]) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, i < w1 && key > T));
        eq += __popc(__ballot_sync(0xffffffffu, i < w1 && key == T));
    }
    if (lane == 0) sm.scan[warp] = (gt << 16) | eq;
    __syncthreads();
    uint32_t ex = 0;
    for (int w = 0; w < warp; ++w) ex += sm.scan[w];
    uint32_t gtb = ex >> 16, eqb = ex & 0xFFFFu;
    const uint32_t r = static_cast<uint32_t>(rem);
    const uint32_t lt = (1u << lane) - 1u;
    for (int b = w0; b < w1; b += 32) {
        const int i = b + lane;
        const uint32_t key = i < w1 ? order_key(sc[i]) : 0u;
        const bool isg = i < w1 && key > T, ise = i < w1 && key == T;
        const uint32_t bg = __ballot_sync(0xffffffffu, isg);
        const uint32_t be = __ballot_sync(0xffffffffu, ise);
        const uint32_t gp = gtb + __popc(bg & lt), ep = eqb + __popc(be & lt);
        int pos = -1;
        if (isg) pos = static_cast<int>(gp + min(ep, r));
        else if (ise && ep < r) pos = static_cast<int>(gp + ep);
        if (pos >= lo && pos < hi) out[pos - lo] = i;
        gtb += __popc(bg);
        eqb += __popc(be);
    }
    __syncthreads();
}

// Entries [lo, hi) of the ascending list of the set bits of
// Long runs of block_extract_bitmap (more than 8 words per warp, over 2048
// scores), kept out of line so that the short path's code is unchanged:
// lane l takes word 32 g + l of the warp's run (g = 0, 1, ...), a prefix
// sum of the words' bit counts over the lanes gives each word's first
// position, and the lane writes the word's set bits in order, those within
// [lo, hi).  `pos`: the set bits of the warps before.
__device__ __noinline__ void extract_bitmap_long(const uint32_t* bitmap, int j0, int j1,
                                                 uint32_t pos, int32_t* out, int lo, int hi) {
    const int lane = threadIdx.x & 31;
    for (int jb = j0; jb < j1 && static_cast<int>(pos) < hi; jb += 32) {
        const int j = jb + lane;
        const uint32_t bits = j < j1 ? bitmap[j] : 0u;
        const uint32_t c = __popc(bits);
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        int at = static_cast<int>(pos + incl - c);
        if (at < hi && at + static_cast<int>(c) > lo) {
            uint32_t b = bits;
            while (b != 0u) {
                const int bit = __ffs(b) - 1;
                b &= b - 1u;
                if (at >= lo && at < hi) out[at - lo] = j * 32 + bit;
                ++at;
            }
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// bitmap[0..nwords), by the whole block: warp w owns the contiguous words
// [w * wpw, (w + 1) * wpw) and wcnt[w] holds the number of set bits in them.
// Each lane places its own bit of every word: position = the set bits of the
// warps before, of the words before in its run, and of the lanes below
// (runs of more than 8 words: extract_bitmap_long).
__device__ __forceinline__ void block_extract_bitmap(const uint32_t* bitmap, int nwords, int wpw,
                                                     const uint32_t* wcnt, int32_t* out, int lo,
                                                     int hi) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t pos = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) pos += w < warp ? wcnt[w] : 0u;
    const int j0 = min(nwords, warp * wpw), j1 = min(nwords, j0 + wpw);
    if (wpw > 8) {
        extract_bitmap_long(bitmap, j0, j1, pos, out, lo, hi);
        return;
    }
    // the run's words read first (independent loads), then placed in order
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t wb[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) wb[u] = j0 + u < j1 ? bitmap[j0 + u] : 0u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint32_t bits = wb[u];
        const int at = static_cast<int>(pos + __popc(bits & lt));
        if (((bits >> lane) & 1u) && at >= lo && at < hi) out[at - lo] = (j0 + u) * 32 + lane;
        pos += __popc(bits);
    }
}

// The warp that owns ballot word wd when warps own runs of wpw words:
// counted against the run starts instead of a division on the select's path.
__device__ __forceinline__ int word_owner(int wd, int wpw) {
    int w = 0;
#pragma unroll
    for (int u = 1; u < kWarps; ++u) w += wd >= u * wpw;
    return w;
}

// Top-k of sc[0..n) (largest scores, ties to the lower index) in ascending
// index order; only list entries [lo, hi) are written, to out[0 .. hi-lo).
// [mn, mx] is the range of the scores.  The kBins histogram bins at the
// start of `scratch` must be zero on entry.  n <= 65535.  Ends with a block
// barrier.
__device__ __forceinline__ void block_topk(const float* sc, int n, int k, float mn, float mx,
                                           int32_t* out, int lo, int hi, uint32_t* scratch,
                                           Small& sm, int stamp_slot) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k >= n) {
        for (int i = max(0, lo) + tid; i < min(n, hi); i += kThreads) out[i - lo] = i;
        __syncthreads();
        return;
    }
    uint32_t* hist = scratch;
    uint32_t* ckey = scratch + kBins;
    int32_t* cidx = reinterpret_cast<int32_t*>(scratch + kBins + kMaxCand);
    uint32_t* inw = scratch + kBins + 2 * kMaxCand;
    // any monotone binning that every CTA computes alike is exact here (the
    // K-th score's bin is then ranked exactly), so a fast division will do
    const float inv = __fdividef(static_cast<float>(kBins), mx - mn);
    if (!(mx > mn)) {                 // every score equal: lowest k indices
        compact_by_threshold(sc, n, order_key(mx), k, out, lo, hi, sm);
        return;
    }
    // the boundary bin from the histogram (block scan, two barriers):
    // sm.misc = {bin, scores still needed from it, its count}; the
    // candidate counter sm.misc[3] reset
    auto find_boundary = [&]() {
        {
            // thread t owns bins 4(255-t) .. 4(255-t)+3 (one 16-byte load);
            // an exclusive scan in thread order counts the scores above them
            const uint4 hv = reinterpret_cast<const uint4*>(hist)[255 - tid];
            const uint32_t tot = hv.x + hv.y + hv.z + hv.w;
            const uint32_t above = block_excl_scan(tot, sm.scan);
            if (above < static_cast<uint32_t>(k) && static_cast<uint32_t>(k) <= above + tot) {
                const uint32_t c[4] = {hv.w, hv.z, hv.y, hv.x};  // descending bins
                uint32_t cum = above;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (cum < static_cast<uint32_t>(k) && static_cast<uint32_t>(k) <= cum + c[j]) {
                        sm.misc[0] = 4 * (255 - tid) + 3 - j;
                        sm.misc[1] = k - static_cast<int>(cum);
                        sm.misc[2] = static_cast<int>(c[j]);
                    }
                    cum += c[j];
                }
            }
            if (tid == 32) sm.misc[3] = 0;
        }
        __syncthreads();
    };
    // exact rank among the m candidates: larger key first, ties to the
    // lower index; the `need` best join the selection (bitmap words and the
    // owning warps' counts); ends with a block barrier
    auto rank_candidates = [&](int m, int need, int wpw) {
        if (m <= 32) {
            if (warp == 0) {
                const uint32_t key = lane < m ? ckey[lane] : 0u;
                const int idx = lane < m ? cidx[lane] : 0x7fffffff;
                int rank = 0;
                // 8 candidates per step, their shuffles independent
                for (int jb = 0; jb < m; jb += 8) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = jb + u;   // < 32 (m <= 32)
                        const uint32_t kj = __shfl_sync(0xffffffffu, key, j);
                        const int ij = __shfl_sync(0xffffffffu, idx, j);
                        rank += j < m && ((kj > key) || (kj == key && ij < idx));
                    }
                }
                if (lane < m && rank < need) {
                    atomicOr(&inw[idx >> 5], 1u << (idx & 31));
                    atomicAdd(&sm.scan[word_owner(idx >> 5, wpw)], 1u);
                }
            }
        } else {
            for (int c = tid; c < m; c += kThreads) {
                const uint32_t key = ckey[c];
                const int idx = cidx[c];
                int rank = 0;
                for (int j = 0; j < m; ++j) {
                    const uint32_t kj = ckey[j];
                    rank += (kj > key) || (kj == key && cidx[j] < idx);
                }
                if (rank < need) {
                    atomicOr(&inw[idx >> 5], 1u << (idx & 31));
                    atomicAdd(&sm.scan[word_owner(idx >> 5, wpw)], 1u);
                }
            }
        }
        __syncthreads();
    };
    if (inv < INFINITY && n <= 8 * kThreads) {
        // Up to 2048 scores: thread t holds scores 8t .. 8t+7 in registers
        // (histogram and selection in one load) and writes byte t of the
        // selection bitmap, so warp w owns words 8w .. 8w+7 and no warp vote
        // is needed; candidates take their slots by one atomic per thread
        // that has any (their order does not matter to the ranking).
        const int i0 = 8 * tid;
        float x[8];
        int bn[8];
        if (i0 + 8 <= n) {
            const float4 a = reinterpret_cast<const float4*>(sc)[2 * tid];
            const float4 b = reinterpret_cast<const float4*>(sc)[2 * tid + 1];
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
            x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
        } else {
#pragma unroll
            for (int v = 0; v < 8; ++v) x[v] = i0 + v < n ? sc[i0 + v] : mn;
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) bn[v] = i0 + v < n ? value_bin(x[v], mn, inv) : -1;
#pragma unroll
        for (int v = 0; v < 8; ++v)
            if (bn[v] >= 0) atomicAdd(&hist[bn[v]], 1u);
        stampk(stamp_slot, 21);                  // this thread's histogram updates issued
        __syncthreads();
        stampk(stamp_slot, 11);                  // histogram done
        find_boundary();
        const int bstar = sm.misc[0], need = sm.misc[1], m = sm.misc[2];
        stampk(stamp_slot, 12);                  // boundary bin known
        if (m <= kMaxCand) {
            const bool all_in = need == m;
            uint32_t selb = 0u, candb = 0u;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int b = bn[v];
                if (b > bstar || (all_in && b == bstar)) selb |= 1u << v;
                else if (b == bstar) candb |= 1u << v;
            }
            reinterpret_cast<uint8_t*>(inw)[tid] = static_cast<uint8_t>(selb);
            const uint32_t cnt = __reduce_add_sync(0xffffffffu, __popc(selb));
            if (lane == 0) sm.scan[warp] = cnt;
            if (candb != 0u) {
                int pos = atomicAdd(&sm.misc[3], __popc(candb));
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    if ((candb >> v) & 1u) {
                        ckey[pos] = order_key(x[v]);
                        cidx[pos] = i0 + v;
                        ++pos;
                    }
                }
            }
            stampk(stamp_slot, 22);              // this thread's bitmap byte out
            __syncthreads();
            stampk(stamp_slot, 13);              // bitmap and candidates out
            if (!all_in) rank_candidates(m, need, 8);
            stampk(stamp_slot, 14);              // boundary candidates ranked
            block_extract_bitmap(inw, (n + 31) / 32, 8, sm.scan, out, lo, hi);
            __syncthreads();
            return;
        }
        __syncthreads();
    } else if (inv < INFINITY) {
        // histogram of the scores over kBins equal bins of [mn, mx] (the
        // bins were zeroed by the caller).  Warp w owns the ballot words
        // [w * wpw, (w + 1) * wpw) (32 scores each) here and in the ballot
        // pass below; the bins of a thread's first 8 words stay in
        // registers for that pass.
        const int nwords = (n + 31) / 32;
        const int wpw = (nwords + kWarps - 1) / kWarps;
        const int j0 = min(nwords, warp * wpw), j1 = min(nwords, j0 + wpw);
        constexpr int V = 8;
        int kbin[V];
        float kx[V];
        for (int jb = j0; jb < j1; jb += V) {
            float x[V];
            int bn[V];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int i = (jb + v) * 32 + lane;
                const bool live = jb + v < j1 && i < n;
                x[v] = live ? sc[i] : mn;
                bn[v] = live ? value_bin(x[v], mn, inv) : -1;
            }
#pragma unroll
            for (int v = 0; v < V; ++v)
                if (bn[v] >= 0) atomicAdd(&hist[bn[v]], 1u);
            if (jb == j0) {
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    kbin[v] = bn[v];
                    kx[v] = x[v];
                }
            }
        }
        stampk(stamp_slot, 21);                  // warp 0's histogram updates issued
        __syncthreads();
        stampk(stamp_slot, 11);                  // histogram done
        find_boundary();
        const int bstar = sm.misc[0], need = sm.misc[1], m = sm.misc[2];
        stampk(stamp_slot, 12);                  // boundary bin known
        if (m <= kMaxCand) {
            // one pass: a ballot word per 32 scores marks those above bin
            // bstar (selected); the scores inside bstar become candidates,
            // all of them selected when the whole bin is needed.  Warp w
            // owns the contiguous words [w * wpw, (w + 1) * wpw) and counts
            // their selected scores.
            const bool all_in = need == m;
            uint32_t cnt = 0;
            for (int jb = j0; jb < j1; jb += V) {
                float x[V];
                int bnv[V];
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int i = (jb + v) * 32 + lane;
                    const bool live = jb + v < j1 && i < n;
                    x[v] = jb == j0 ? kx[v] : (live ? sc[i] : mn);
                    bnv[v] = jb == j0 ? kbin[v] : (live ? value_bin(x[v], mn, inv) : -1);
                }
                uint32_t cw[V];     // candidates (scores in bin bstar) of each word
                uint32_t ncand = 0;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int wd = jb + v;
                    const int i = wd * 32 + lane;
                    const bool live = wd < j1 && i < n;
                    const int bn = bnv[v];
                    const uint32_t gw =
                        __ballot_sync(0xffffffffu, live && (bn > bstar || (all_in && bn == bstar)));
                    if (lane == 0 && wd < j1) inw[wd] = gw;
                    cnt += __popc(gw);
                    cw[v] = all_in ? 0u : __ballot_sync(0xffffffffu, live && bn == bstar);
                    ncand += __popc(cw[v]);
                }
                if (ncand != 0) {
                    // one slot reservation per warp and chunk, then each
                    // candidate lane writes at its place
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&sm.misc[3], static_cast<int>(ncand));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        if ((cw[v] >> lane) & 1u) {
                            const int pos = base + __popc(cw[v] & lt);
                            ckey[pos] = order_key(x[v]);
                            cidx[pos] = (jb + v) * 32 + lane;
                        }
                        base += __popc(cw[v]);
                    }
                }
            }
            if (lane == 0) sm.scan[warp] = cnt;
            stampk(stamp_slot, 22);              // warp 0's ballot words out
            __syncthreads();
            stampk(stamp_slot, 13);              // ballot words and candidates out
            if (!all_in) rank_candidates(m, need, wpw);
            stampk(stamp_slot, 14);              // boundary candidates ranked
            block_extract_bitmap(inw, nwords, wpw, sm.scan, out, lo, hi);
            __syncthreads();
            return;
        }
        __syncthreads();
    }
    uint32_t T = 0;
    int rem = 0;
    radix_threshold(sc, n, k, scratch, sm, &T, &rem);
    compact_by_threshold(sc, n, T, rem, out, lo, hi, sm);
}

#ifndef ABSP_DECODE_MIN_BLOCKS
#define ABSP_DECODE_MIN_BLOCKS 2  // CTAs per SM the register budget is built for
#endif

// DIAG: the failure-path diagnostic (ABSP_STEP_DIAG_WAIT_TIMEOUT): the
// score barrier expects 16 bytes that are never sent and every bounded wait
// gives up after 1 ms, so the score wait runs out, records ABSP_ERR_TIMEOUT
// and the kernel carries on to its normal end.
template <int MODE, bool BIG_GROUP, bool EARLY, bool BF16C, bool GM, bool DIAG, int NPB>
__global__ void __launch_bounds__(kThreads, NPB == 2 ? 1 : ABSP_DECODE_MIN_BLOCKS)
    decode_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the shared array by a byte offset
    // so that every access below stays in the shared address space
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* regB = base;                        // scores + ring / pages / warp merge
    uint8_t* regA = base + p.regA_off;           // cluster merge receive buffers
    Small& sm = *reinterpret_cast<Small*>(base + p.small_off);
    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(base + p.qs_off);  // [G][128]
    int32_t* sel_s = reinterpret_cast<int32_t*>(base + p.qs_off + p.kv.G * kD * 2);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    stampk(p.stamp_slot, 0);                     // entry
    const uint32_t C = cluster_nctarank();
    const uint32_t rank = cluster_ctarank();
    // C (a power of two), bs and bs / 16 are powers of two: shifts, not
    // divisions, on the dependent path
    const int lgC = __ffs(static_cast<int>(C)) - 1;
    const int pair = blockIdx.x >> lgC;
    const int Hkv = p.kv.Hkv, G = p.kv.G;
    const int s = pair / Hkv, h = pair % Hkv;
    const int bs = p.kv.bs[h];
    const int spb = bs / kPage;
    const int32_t* pt = p.kv.page_table + static_cast<int64_t>(s) * p.kv.max_pages;
    constexpr bool kSelect = (MODE & kModeSelect) != 0;
    constexpr bool kAttend = (MODE & kModeAttend) != 0;
    // centroid rows: 64 B of INT4 codes, or 256 B of bf16 centroids
    constexpr int kRow = BF16C ? 2 * kD : kRowBytes;
    constexpr int kSRows = kStageBytes / kRow;         // rows per bulk stage
    constexpr uint64_t kWaitNs = DIAG ? 1000000ull : kWaitLimitNs;

    if constexpr (kAttend) {
        // the page copies' tensor-map descriptors, fetched ahead of the
        // first copy (they are kernel parameters, not produced by the
        // preceding kernel)
        if (tid == 32) {
            prefetch_tensormap(&tmk);
            prefetch_tensormap(&tmv);
        }
    }
    if (tid == 0) {
        for (int i = 0; i < kMaxStages; ++i) mbar_init(smem_u32(&sm.bar_code[i]), 1);
        for (int w = 0; w < 2 * kWarps; ++w) mbar_init(smem_u32(&sm.bar_page[w]), 1);
        mbar_init(smem_u32(&sm.bar_score), 1);
        mbar_init(smem_u32(&sm.bar_merge), 1);
        fence_mbar_init();
    }
    // Without EARLY nothing in global memory is read before this wait.
    if constexpr (!EARLY) {
        pdl_wait();
        pdl_trigger();
    }
    int len = p.kv.seq_lens[s];
    if (len < 0 || len > p.kv.max_pages * kPage) {
        if (tid == 0 && rank == 0 && h == 0) set_error(p.err, ABSP_ERR_DEVICE_FAULT, s);
        len = 0;
    }
    const int lgbs = __ffs(bs) - 1, lgspb = lgbs - 4;
    const int n = (len + bs - 1) >> lgbs;
    // rows of this CTA: a contiguous range, a multiple of 4 rows long
    const int per = (((n + static_cast<int>(C) - 1) >> lgC) + 3) & ~3;
    const int r0 = min(n, static_cast<int>(rank) * per);
    const int nrows = min(n, r0 + per) - r0;
    const int nchunks = (nrows + kSRows - 1) / kSRows;
    const int npg = (len + kPage - 1) / kPage;
    // The selected blocks' page ids: in the fused mode each CTA stages the
    // page-table entries of its own scored rows in shared memory and the
    // attending CTAs read them through distributed shared memory, when the
    // slice fits and every warp attends at most 32 pages (all lookups then
    // happen once, at the start of the attention, while every CTA of the
    // cluster is still running: none leaves before it received every other
    // CTA's merge partial).  Uniform over a cluster.
    const int Ksel = min(n, max(1, p.budget >> lgbs));
    // Preferred: every CTA stages the sequence's whole page-table row in its
    // own shared memory (asynchronous 4-byte copies issued here, before the
    // dependency wait with early prefetch), so that a page id is one local
    // read.  When the row does not fit, the own-rows slices below.
    int32_t* ptrow = reinterpret_cast<int32_t*>(base + p.ptrow_off);
    const bool stage_row = kSelect && kAttend && npg <= p.pt_cap;
    if (stage_row) {
        for (int i = tid; i < npg; i += kThreads) cp_async_4(smem_u32(ptrow + i), pt + i);
        cp_async_commit();
    }
    const bool stage_pt = kSelect && kAttend && !stage_row && per > 0 && per * spb <= kPtStage &&
                          ((Ksel * spb + static_cast<int>(C) - 1) >> lgC) <= 32 * kWarps;
    int ptv[kPtStage / kThreads];
#pragma unroll
    for (int u = 0; u < kPtStage / kThreads; ++u) {
        const int i = tid + u * kThreads;
        const int lp = r0 * spb + i;
        ptv[u] = stage_pt && i < nrows * spb && lp < npg ? pt[lp] : -1;
    }
    const uint8_t* cbase =
        p.codes + (static_cast<int64_t>(s) * p.kv.rows_per_seq + p.kv.row_base[h] + r0) * kRow;
    // code ring: region B past the scores and select scratch (region B is
    // free for it until the attention phase)
    const int NS = p.nstages;
    auto stage_buf = [&](int st) -> uint8_t* { return regB + p.ring_off + st * kStageBytes; };
    if (tid == 0) {
        if (kAttend && C > 1)
            // every CTA's slice of its partial, this one's own included:
            // G rows x 128/C channels, and (M, L) per row
            mbar_arrive_expect_tx(smem_u32(&sm.bar_merge), C * (G * (kD / C) * 4 + 8 * G));
        if (kSelect && (MODE != kModeSelect || rank == 0))
            // every CTA's scores but this one's own (plain stores), and
            // every CTA's (min, max)
            mbar_arrive_expect_tx(smem_u32(&sm.bar_score),
                                  16 * ((n + 3) / 4 - (nrows + 3) / 4) + 8 * C + (DIAG ? 16 : 0));
        if (kSelect) {
            for (int c = 0; c < min(nchunks, NS); ++c) {
                const int rows = min(kSRows, nrows - c * kSRows);
                const uint32_t bar = smem_u32(&sm.bar_code[c]);
                mbar_arrive_expect_tx(bar, rows * kRow);
                bulk_g2s(smem_u32(stage_buf(c)), cbase + c * kStageBytes, rows * kRow, bar);
            }
            // the stages past the ring come from L2 when the ring refills
            for (int c = NS; c < nchunks; ++c)
                bulk_prefetch_l2(cbase + c * kStageBytes,
                                 static_cast<uint32_t>(min(kSRows, nrows - c * kSRows) * kRow));
        }
    }
    if constexpr (kSelect) {
        // the select's histogram bins (in region B's select scratch, which
        // nothing touches before the select), zeroed ahead of the wait
        uint32_t* hist = reinterpret_cast<uint32_t*>(regB + p.scratch_off);
        for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
    }
    // B0 arrive (release: the barrier set-up above is visible cluster-wide
    // once B0 completes); matched by the wait before the first remote access.
    cluster_arrive();
    if (kAttend && !stage_pt && !stage_row) {
        // the attention phase reads page-table entries of this sequence
        for (int i = tid * 32; i < npg; i += kThreads * 32) prefetch_l2(pt + i);
    }
    float scl = 0.0f;
    int32_t zpv = 0;
    if (kSelect && tid < kD) {
        const int64_t pi = (static_cast<int64_t>(s) * Hkv + h) * kD + tid;
        if constexpr (!BF16C) {
            scl = p.scale[pi];
            zpv = p.zp[pi];
        }
    }
    if constexpr (EARLY && kSelect) {
        // an L2 hint for the group's queries (read below, after the wait;
        // when the preceding kernel writes them, its writes land in L2 and
        // the read sees them, as it would without this hint)
        if (tid < G * kD * 2 / 128)
            prefetch_l2(reinterpret_cast<const uint8_t*>(
                            p.q + (static_cast<int64_t>(s) * p.kv.Hq + h * G) * kD) + tid * 128);
    }
    if constexpr (EARLY) {
        // B0 only needs the cluster's CTAs to have started: wait for it while
        // the preceding kernel still runs.  Only the query may be produced
        // by the preceding kernel.
        cluster_wait();
        pdl_wait();
        pdl_trigger();
    }
    stampk(p.stamp_slot, 1);                     // released by the preceding launch
    int K = 0;
    int sel_lo = 0, sel_hi = 0;  // list entries held in sel_s

    if constexpr (kSelect) {
        // ---------------------------------------------------- A: score --
        K = Ksel;
        if (stage_pt) {
#pragma unroll
            for (int u = 0; u < kPtStage / kThreads; ++u) sm.pt[tid + u * kThreads] = ptv[u];
        }
        if (stage_row) cp_async_wait_all();   // this thread's copies; the barrier below
                                              // makes the whole row visible
        if (tid < kD) {
            const __nv_bfloat16* qh = p.q + (static_cast<int64_t>(s) * p.kv.Hq + h * G) * kD + tid;
            // the group's queries are read once (they may live in host
            // memory), all loads issued before the first use, and kept for
            // the attention phase; qbar sums them in head order
            constexpr int kQMax = BIG_GROUP ? 16 : 8;
            __nv_bfloat16 qv[kQMax];
#pragma unroll
            for (int j = 0; j < kQMax; ++j) qv[j] = j < G ? qh[j * kD] : __float2bfloat16(0.0f);
            float qb = 0.0f;
#pragma unroll
            for (int j = 0; j < kQMax; ++j) {
                if (j < G) {
                    qs[j * kD + tid] = qv[j];
                    qb += __bfloat162float(qv[j]);
                }
            }
            const float wv = BF16C ? qb : qb * scl;
            sm.w[tid] = wv;
            sm.zb[tid] = 8388608.0f + static_cast<float>(zpv);
            sm.zf[tid] = static_cast<float>(zpv);
            if constexpr (!BF16C && !GM) {
                // INT4 sum scores: sum_ch w (code - zp) = sum_ch w code -
                // sum_ch w zp.  Lane group `sub` (channels 16 sub .. 16 sub
                // + 15, the 16 threads tid & ~15 here) works at scale 2^-X,
                // X from its largest |w| (2^e <= max|w| < 2^(e+1)): the
                // pre-scaled weights w 2^(149 - 4j - X) stay below 2^126 and
                // products of the larger weights are normal.  Each thread
                // prepares its channel once for the 32 lanes that use it.
                float mw = fabsf(wv), zs = wv * static_cast<float>(zpv);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) {
                    mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
                    zs += __shfl_xor_sync(0xffffffffu, zs, o);
                }
                const int e = static_cast<int>((__float_as_uint(mw) >> 23) & 0xFFu) - 127;
                const int X = min(126, max(22, 24 + e));
                sm.w[tid] = wv * __uint_as_float(static_cast<uint32_t>(276 - X - 4 * (tid & 3)) << 23);
                if ((tid & 15) == 0) {
                    sm.kz[tid >> 4] = zs * __uint_as_float(static_cast<uint32_t>(127 - X) << 23);
                    sm.xs[tid >> 4] = __uint_as_float(static_cast<uint32_t>(127 + X) << 23);
                }
            }
            if constexpr (GM) {
                float* wg = reinterpret_cast<float*>(regB + p.wg_off);
                const int slot = (tid >> 4) * 20 + (tid & 15);
                for (int j = 0; j < G; ++j) {
                    const float qj = __bfloat162float(qs[j * kD + tid]);
                    wg[j * kWgStride + slot] = BF16C ? qj : qj * scl;
                }
            }
        }
        __syncthreads();
        stampk(p.stamp_slot, 2);                 // query and weights ready
        const int sub = tid & 7, grp = tid >> 3;  // 32 groups of 8 lanes
        float wr[16], zr[16];
        float kz = 0.0f;  // this lane's share of sum_ch w[ch] * zp[ch], scaled
        float xs = 1.0f;  // 2^X: undoes the lane's scale on its partial sum
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            const float4 v = *reinterpret_cast<const float4*>(&sm.w[sub * 16 + 4 * k4]);
            wr[4 * k4] = v.x;
            wr[4 * k4 + 1] = v.y;
            wr[4 * k4 + 2] = v.z;
            wr[4 * k4 + 3] = v.w;
        }
        if constexpr (GM) {
#pragma unroll
            for (int k = 0; k < 16; ++k) zr[k] = sm.zb[sub * 16 + k];
        }
        if constexpr (!BF16C && !GM) {
            kz = sm.kz[sub];
            xs = sm.xs[sub];
        }
        float* scores = reinterpret_cast<float*>(regB);
        const uint32_t scores_u32 = smem_u32(scores);
        const uint32_t bar_score = smem_u32(&sm.bar_score);
        float lmin = INFINITY, lmax = -INFINITY;
        if constexpr (!EARLY) cluster_wait();  // B0: every CTA of the cluster is running
        stampk(p.stamp_slot, 18);                // scoring starts
        // The chunk loop over the code ring; score4(sbuf, r4, rows) gives one
        // 8-lane group's scores of rows r4 .. r4 + 3 of a stage (values for
        // rows past `rows` are discarded here).
        auto chunk_loop = [&](auto&& score4) {
            // ring stage and mbarrier phase of chunk c, counted (NS is a
            // launch value: a division here sat on the critical path)
            int stage = 0, phase = 0;
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                mbar_wait_bounded(smem_u32(&sm.bar_code[stage]), phase, p.err, 1, kWaitNs);
                if (c == 0) stampk(p.stamp_slot, 19);  // first code stage here
                const int rows = min(kSRows, nrows - c * kSRows);
                const uint8_t* sbuf = stage_buf(stage);
#pragma unroll 1
                for (int rb = 0; rb < rows; rb += 4 * (kThreads / 8)) {
                    const int r4 = rb + 4 * grp;
                    const float4 q = score4(sbuf, r4, rows);
                    float q4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (r4 + u < rows) {
                            lmin = fminf(lmin, q4[u]);
                            lmax = fmaxf(lmax, q4[u]);
                        } else {
                            q4[u] = 0.0f;
                        }
                    }
                    if (r4 < rows) {
                        // to this CTA by a plain store, to the others by
                        // st.async (which counts the bytes on their mbarrier)
                        const uint32_t off = 4u * static_cast<uint32_t>(r0 + c * kSRows + r4);
                        for (uint32_t dst = sub; dst < (MODE == kModeSelect ? 1u : C); dst += 8) {
                            if (dst == rank)
                                *reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(scores) + off) =
                                    make_float4(q4[0], q4[1], q4[2], q4[3]);
                            else
                                st_async_v4(dsmem_addr(scores_u32 + off, dst), q4[0], q4[1], q4[2],
                                            q4[3], dsmem_addr(bar_score, dst));
                        }
                    }
                }
                if (c == 0) stampk(p.stamp_slot, 20);  // warp 0 scored the first stage
                // a stage buffer is refilled once every warp is done with it
                // (uniform); the block barrier after the loop, before the
                // scores are read, covers the stages that are not refilled
                if (c + NS < nchunks) {
                    __syncthreads();
                    if (tid == 0) {
                        const int cn = c + NS;
                        const int rows_n = min(kSRows, nrows - cn * kSRows);
                        const uint32_t bar = smem_u32(&sm.bar_code[stage]);
                        fence_proxy_async_smem();
                        mbar_arrive_expect_tx(bar, rows_n * kRow);
                        bulk_g2s(smem_u32(sbuf), cbase + cn * kStageBytes, rows_n * kRow, bar);
                    }
                }
                if (++stage == NS) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        };
        // The variant is uniform over the launch: each gets its own loop, so
        // the four rows of a group are independent chains (no branch between
        // them) and their sums take one transpose-reduction.
        if constexpr (!GM) {
            if constexpr (BF16C) {
                chunk_loop([&](const uint8_t* sbuf, int r4, int rows) {
                    float a[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        // 16 bf16 centroid channels per lane: score += qbar * c
                        uint4 y0 = make_uint4(0u, 0u, 0u, 0u), y1 = y0;
                        if (r4 + u < rows) {
                            const uint4* src =
                                reinterpret_cast<const uint4*>(sbuf + (r4 + u) * kRow + sub * 32);
                            y0 = src[0];
                            y1 = src[1];
                        }
                        const uint32_t yy[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
                        float acc = 0.0f;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            acc = fmaf(wr[2 * k], bf16lo(yy[k]), acc);
                            acc = fmaf(wr[2 * k + 1], bf16hi(yy[k]), acc);
                        }
                        a[u] = acc;
                    }
                    return group_sum4(a, lane);
                });
            } else {
                chunk_loop([&](const uint8_t* sbuf, int r4, int rows) {
                    float a[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint2 x = make_uint2(0u, 0u);
                        if (r4 + u < rows)
                            x = *reinterpret_cast<const uint2*>(sbuf + (r4 + u) * kRow + sub * 8);
                        a[u] = int4_dot16(x, wr, -kz) * xs;
                    }
                    return group_sum4(a, lane);
                });
            }
        } else {
            chunk_loop([&](const uint8_t* sbuf, int r4, int rows) {
                float sc[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = r4 + u;
                    float acc;
                    // variant: the largest of the group's per-head scores
                    float f[16];
                    if constexpr (BF16C) {
                        uint4 y0 = make_uint4(0u, 0u, 0u, 0u), y1 = y0;
                        if (r < rows) {
                            const uint4* src =
                                reinterpret_cast<const uint4*>(sbuf + r * kRow + sub * 32);
                            y0 = src[0];
                            y1 = src[1];
                        }
                        const uint32_t yy[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            f[2 * k] = bf16lo(yy[k]);
                            f[2 * k + 1] = bf16hi(yy[k]);
                        }
                    } else {
                        uint2 x = make_uint2(0u, 0u);
                        if (r < rows)
                            x = *reinterpret_cast<const uint2*>(sbuf + r * kRow + sub * 8);
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            f[k] = __uint_as_float(0x4B000000u | ((x.x >> (4 * k)) & 0xFu)) - zr[k];
                            f[8 + k] =
                                __uint_as_float(0x4B000000u | ((x.y >> (4 * k)) & 0xFu)) - zr[8 + k];
                        }
                    }
                    const float* wg = reinterpret_cast<const float*>(regB + p.wg_off) + sub * 20;
                    acc = -INFINITY;
                    for (int jh = 0; jh < G; ++jh) {
                        const float4* w4 = reinterpret_cast<const float4*>(wg + jh * kWgStride);
                        float a = 0.0f;
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const float4 wv = w4[k4];
                            a = fmaf(wv.x, f[4 * k4], a);
                            a = fmaf(wv.y, f[4 * k4 + 1], a);
                            a = fmaf(wv.z, f[4 * k4 + 2], a);
                            a = fmaf(wv.w, f[4 * k4 + 3], a);
                        }
                        a += __shfl_xor_sync(0xffffffffu, a, 1);
                        a += __shfl_xor_sync(0xffffffffu, a, 2);
                        a += __shfl_xor_sync(0xffffffffu, a, 4);
                        acc = fmaxf(acc, a);
                    }
                    sc[u] = acc;
                }
                return make_float4(sc[0], sc[1], sc[2], sc[3]);
            });
        }
        stampk(p.stamp_slot, 3);                 // own rows scored
        // this CTA's score range, sent along with the scores
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lmin = fminf(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
            lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        }
        if (lane == 0) {
            sm.red[0][warp] = lmin;
            sm.red[1][warp] = lmax;
        }
        __syncthreads();
        if (tid < static_cast<int>(C) && (MODE != kModeSelect || tid == 0)) {
            float a = sm.red[0][0], b = sm.red[1][0];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) {
                a = fminf(a, sm.red[0][w]);
                b = fmaxf(b, sm.red[1][w]);
            }
            st_async_v2(dsmem_addr(smem_u32(&sm.cmm[rank]), tid), a, b,
                        dsmem_addr(bar_score, tid));
        }
        // select-only: CTA 0 alone receives and selects
        if (MODE == kModeSelect && rank != 0) return;
        // ------------------------------------- B: every score arrived --
        mbar_wait_bounded<true>(bar_score, 0, p.err, 4, kWaitNs);
        stampk(p.stamp_slot, 4);                 // every CTA's scores here
        if (kAttend && tid == 32) {
            // the copies' descriptors again, a top-K ahead of the first copy
            // (fetched at entry, which can be microseconds earlier)
            prefetch_tensormap(&tmk);
            prefetch_tensormap(&tmv);
        }

        // --------------------------------------------------- C: select --
        float2 rv[16];                       // C <= 16: a tree, not a chain
#pragma unroll
        for (uint32_t r = 0; r < 16; ++r) rv[r] = r < C ? sm.cmm[r] : make_float2(INFINITY, -INFINITY);
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
            for (int r = 0; r < w; ++r) {
                rv[r].x = fminf(rv[r].x, rv[r + w].x);
                rv[r].y = fmaxf(rv[r].y, rv[r + w].y);
            }
        }
        const float smin = rv[0].x, smax = rv[0].y;
        // this CTA attends list entries [sel_lo, sel_hi): the blocks of its
        // share [ppb, ppe) of the K * bs/16 selected pages
        const int Pp = K * spb;
        const int ppb = static_cast<int>((static_cast<uint32_t>(Pp) * rank) >> lgC);  // P*C < 2^21
        const int ppe = static_cast<int>((static_cast<uint32_t>(Pp) * (rank + 1)) >> lgC);
        if (MODE == kModeSelect) {
            sel_lo = 0;
            sel_hi = K;
        } else {
            sel_lo = ppb >> lgspb;
            sel_hi = ppe > ppb ? ((ppe - 1) >> lgspb) + 1 : sel_lo;
        }
        block_topk(scores, n, K, smin, smax, sel_s, sel_lo, sel_hi,
                   reinterpret_cast<uint32_t*>(regB + p.scratch_off), sm, p.stamp_slot);
        stampk(p.stamp_slot, 5);                 // top-K done
        if (MODE == kModeSelect) {
            int32_t* dst = p.sel + (static_cast<int64_t>(s) * Hkv + h) * p.kmax;
            for (int i = tid; i < K; i += kThreads) dst[i] = sel_s[i];  // [0, K) held
            if (tid == 0) p.sel_count[static_cast<int64_t>(s) * Hkv + h] = K;
            return;
        }
    } else {
        // read a selection made by a separate score/select call
        K = p.sel_count[static_cast<int64_t>(s) * Hkv + h];
        if (K < 0 || K > p.kmax) {
            if (tid == 0 && rank == 0) set_error(p.err, ABSP_ERR_DEVICE_FAULT, s);
            K = 0;
        }
        const int32_t* src = p.sel + (static_cast<int64_t>(s) * Hkv + h) * p.kmax;
        for (int i = tid; i < K; i += kThreads) {
            int b = src[i];
            if (b < 0 || b >= n) {
                set_error(p.err, ABSP_ERR_DEVICE_FAULT, s);
                b = -1;
            }
            sel_s[i] = b;
        }
        __syncthreads();
    }

    if constexpr ((MODE & kModeAttend) != 0) {
        // --------------------------------------------------- D: attend --
        const int P = K * spb;
        const int pb = static_cast<int>((static_cast<uint32_t>(P) * rank) >> lgC);  // P*C < 2^21
        const int pe = static_cast<int>((static_cast<uint32_t>(P) * (rank + 1)) >> lgC);
        const int cnt_w = pe - pb > warp ? (pe - pb - warp + kWarps - 1) / kWarps : 0;
        const int g = lane >> 2, t4 = lane & 3;
        // queries: the copy made while scoring; attend-only launches make it
        // here (the query is 4-byte aligned)
        if constexpr (!kSelect) {
            const uint32_t* qsrc = reinterpret_cast<const uint32_t*>(
                p.q + (static_cast<int64_t>(s) * p.kv.Hq + h * G) * kD);
            for (int i = tid; i < G * kD / 2; i += kThreads)
                reinterpret_cast<uint32_t*>(qs)[i] = qsrc[i];
            __syncthreads();
        }
        const __nv_bfloat16* qg = qs;
        float o[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
        float m0 = -FLT_MAX, m8 = -FLT_MAX, l0 = 0.0f, l8 = 0.0f;
        bool any0 = false;  // this warp has seen at least one valid token
        const float qks = p.qk_scale_log2;
        // this warp's page buffers: page i goes to buffer i % NPB
        constexpr int npbuf = NPB;
        uint8_t* wbuf = regB + warp * npbuf * kPageSmem;

        // Pages of this warp, 32 at a time: lane l resolves page c0 + l into
        // its physical page id and valid token count (one parallel round of
        // page-table reads instead of one read per page); a page that is
        // past the sequence end, or whose id is out of range, gets 0 tokens.
        int my_phys = 0, my_valid = 0, c0 = 0;
        auto resolve = [&](int i0) {
            c0 = i0;
            my_phys = 0;
            my_valid = 0;
            const int i = i0 + lane;
            if (i >= cnt_w) return;
            const int j = pb + warp + kWarps * i;
            const int b = sel_s[(j >> lgspb) - sel_lo];
            if (b < 0) return;
            const int lp = b * spb + (j & (spb - 1));
            const int valid = min(kPage, len - lp * kPage);
            if (valid <= 0) return;
            int phys;
            if (stage_row) {
                phys = ptrow[lp];
            } else if (stage_pt) {
                // staged by the CTA that scored block b
                // b / per by a float reciprocal, corrected to the exact
                // quotient (b < 2^14, per >= 4)
                int owner = __float2int_rz((static_cast<float>(b) + 0.5f) *
                                           __frcp_rn(static_cast<float>(per)));
                owner += (owner + 1) * per <= b;
                owner -= owner * per > b;
                int32_t* e = &sm.pt[lp - owner * per * spb];
                phys = owner == static_cast<int>(rank) ? *e
                                                        : dsmem_ld_s32(dsmem_addr(smem_u32(e), owner));
            } else {
                phys = pt[lp];
            }
            if (phys < 0 || phys >= p.kv.num_phys_pages) {
                set_error(p.err, ABSP_ERR_DEVICE_FAULT, s);
                return;
            }
            my_phys = phys;
            my_valid = valid;
        };

        // page i of this warp: tensor copies of its K and V slices (every
        // lane calls this; lane 0 issues).  The caller has ordered this
        // lane's earlier generic accesses of the buffer before the copy
        // (fence.proxy.async after the warp's last use of it).
        auto issue = [&](int i) -> int {
            if (i >= c0 + 32) resolve(i);
            const int valid = __shfl_sync(0xffffffffu, my_valid, i & 31);
            const int phys = __shfl_sync(0xffffffffu, my_phys, i & 31);
            if (lane == 0) {
                const int k = i & (npbuf - 1);
                const uint32_t bar = smem_u32(&sm.bar_page[2 * warp + k]);
                mbar_arrive_expect_tx(bar, valid > 0 ? kPageSmem : 0);
                if (valid > 0) {
                    const int y = (phys * Hkv + h) * kPage;
                    const uint32_t dst = smem_u32(wbuf + k * kPageSmem);
                    tma_load_2d(dst, &tmk, 0, y, bar);
                    tma_load_2d(dst + 2048, &tmk, 64, y, bar);
                    tma_load_2d(dst + 4096, &tmv, 0, y, bar);
                    tma_load_2d(dst + 6144, &tmv, 64, y, bar);
                }
            }
            return valid;
        };

        // page i of this warp into L2 ahead of its copy, when it is among
        // the pages resolved (every lane calls this; lane 0 issues)
        auto prefetch = [&](int i) {
            if (i >= cnt_w || i < c0 || i >= c0 + 32) return;
            const int valid = __shfl_sync(0xffffffffu, my_valid, i & 31);
            const int phys = __shfl_sync(0xffffffffu, my_phys, i & 31);
            if (lane != 0 || valid <= 0) return;
            const int64_t off = (static_cast<int64_t>(phys) * Hkv + h) * (kPage * kD);
            bulk_prefetch_l2(p.kv.k_pages + off, kPage * kD * 2);
            bulk_prefetch_l2(p.kv.v_pages + off, kPage * kD * 2);
        };

        // (the select, or the copy of a given selection, ended with a barrier:
        // no thread reads the scores in region B any more)
        stampk(p.stamp_slot, 16);
        resolve(0);
        stampk(p.stamp_slot, 17);                // page ids of the first 32 pages
        // the valid token counts of the pages in flight, by buffer (the
        // buffers held scores and select scratch before the barrier that
        // ended the select: one proxy fence orders those accesses before
        // the first copies)
        fence_proxy_async_smem();
        __syncwarp();
        stampk(p.stamp_slot, 23);                // proxy fence passed
        int vbuf0 = cnt_w > 0 ? issue(0) : 0;
        int vbuf1 = npbuf == 2 && cnt_w > 1 ? issue(1) : 0;
        stampk(p.stamp_slot, 15);                // first page copies issued
#pragma unroll 1
        for (int i = 1; i <= ABSP_PAGE_PREFETCH; ++i) prefetch(i);
#pragma unroll 1
        for (int i = 0; i < cnt_w; ++i) {
            const int k = i & (npbuf - 1);
            const int valid = k ? vbuf1 : vbuf0;
            mbar_wait_bounded(smem_u32(&sm.bar_page[2 * warp + k]), (i >> (npbuf - 1)) & 1, p.err,
                              2, kWaitNs);
            if (i == 0) stampk(p.stamp_slot, 6);  // warp 0's first page landed
            if (valid > 0) {
                uint8_t* pg = wbuf + k * kPageSmem;
                const uint32_t kb = smem_u32(pg), vb = kb + 4096;
                if (valid < kPage) {
                    // zero the V rows past the sequence end (they may hold
                    // anything, including NaN); each row is 128 B per half
                    const int nz = (kPage - valid) * 16;  // 16-byte chunks
                    for (int c = lane; c < nz; c += 32) {
                        const int row = valid + (c >> 4);
                        const int half = (c >> 3) & 1;
                        *reinterpret_cast<uint4*>(pg + 4096 + half * 2048 + row * 128 + (c & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    __syncwarp();
                }
                // S^T[row][token] = sum_d Q[row][d] K[token][d], 16 tokens
                float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
                const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t kh = kb + (j >> 2) * 2048;
                    const int tok = (mi >> 1) * 8 + ri;
                    const int ch = (j & 3) * 2 + (mi & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kh + tok * 128 + ((ch ^ ri) << 4), b0, b1, b2, b3);
                    // the query fragments are re-read from shared memory at
                    // each use rather than held through the page loop: no
                    // kernel spills at 128 registers (two CTAs per SM)
                    const uint32_t qx = g < G ? ld_u32(qg + g * kD + 16 * j + 2 * t4) : 0u;
                    const uint32_t qy = g < G ? ld_u32(qg + g * kD + 16 * j + 8 + 2 * t4) : 0u;
                    if constexpr (BIG_GROUP) {
                        const uint32_t qz =
                            g + 8 < G ? ld_u32(qg + (g + 8) * kD + 16 * j + 2 * t4) : 0u;
                        const uint32_t qw =
                            g + 8 < G ? ld_u32(qg + (g + 8) * kD + 16 * j + 8 + 2 * t4) : 0u;
                        mma_bf16(s0[0], s0[1], s0[2], s0[3], qx, qz, qy, qw, b0, b1);
                        mma_bf16(s1[0], s1[1], s1[2], s1[3], qx, qz, qy, qw, b2, b3);
                    } else {
                        mma_bf16_top(s0[0], s0[1], qx, qy, b0, b1);
                        mma_bf16_top(s1[0], s1[1], qx, qy, b2, b3);
                    }
                }
                // scale to log2 units and mask tokens past the end
                const int ta = 2 * t4, tb = 8 + 2 * t4;
                const float x0 = ta < valid ? s0[0] * qks : -INFINITY;
                const float x1 = ta + 1 < valid ? s0[1] * qks : -INFINITY;
                const float x2 = tb < valid ? s1[0] * qks : -INFINITY;
                const float x3 = tb + 1 < valid ? s1[1] * qks : -INFINITY;
                float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                // valid >= 1 so token 0 is valid: mx is finite
                const float mn0 = fmaxf(m0, mx);
                const float corr0 = any0 ? fast_exp2(m0 - mn0) : 0.0f;
                const uint32_t pa0 = pack_bf16x2(fast_exp2(x0 - mn0), fast_exp2(x1 - mn0));
                const uint32_t pa2 = pack_bf16x2(fast_exp2(x2 - mn0), fast_exp2(x3 - mn0));
                l0 = l0 * corr0 + (bf16lo(pa0) + bf16hi(pa0) + bf16lo(pa2) + bf16hi(pa2));
                m0 = mn0;
                uint32_t pa1 = 0u, pa3 = 0u;
                float corr8 = 1.0f;
                if constexpr (BIG_GROUP) {
                    const float y0 = ta < valid ? s0[2] * qks : -INFINITY;
                    const float y1 = ta + 1 < valid ? s0[3] * qks : -INFINITY;
                    const float y2 = tb < valid ? s1[2] * qks : -INFINITY;
                    const float y3 = tb + 1 < valid ? s1[3] * qks : -INFINITY;
                    float my = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
                    my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, 1));
                    my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, 2));
                    const float mn8 = fmaxf(m8, my);
                    corr8 = any0 ? fast_exp2(m8 - mn8) : 0.0f;
                    pa1 = pack_bf16x2(fast_exp2(y0 - mn8), fast_exp2(y1 - mn8));
                    pa3 = pack_bf16x2(fast_exp2(y2 - mn8), fast_exp2(y3 - mn8));
                    l8 = l8 * corr8 + (bf16lo(pa1) + bf16hi(pa1) + bf16lo(pa3) + bf16hi(pa3));
                    m8 = mn8;
                }
                if (any0) {   // nothing to rescale before this warp's first valid page
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        o[t][0] *= corr0;
                        o[t][1] *= corr0;
                        if constexpr (BIG_GROUP) {
                            o[t][2] *= corr8;
                            o[t][3] *= corr8;
                        }
                    }
                }
                any0 = true;
                // O[row][d] += P[row][token] V[token][d]
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const uint32_t vh = vb + (cc >> 2) * 2048;
                    const int tok = (mi & 1) * 8 + ri;
                    const int ch = (cc & 3) * 2 + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(vh + tok * 128 + ((ch ^ ri) << 4), b0, b1, b2, b3);
                    if constexpr (BIG_GROUP) {
                        mma_bf16(o[2 * cc][0], o[2 * cc][1], o[2 * cc][2], o[2 * cc][3], pa0, pa1,
                                 pa2, pa3, b0, b1);
                        mma_bf16(o[2 * cc + 1][0], o[2 * cc + 1][1], o[2 * cc + 1][2],
                                 o[2 * cc + 1][3], pa0, pa1, pa2, pa3, b2, b3);
                    } else {
                        mma_bf16_top(o[2 * cc][0], o[2 * cc][1], pa0, pa2, b0, b1);
                        mma_bf16_top(o[2 * cc + 1][0], o[2 * cc + 1][1], pa0, pa2, b2, b3);
                    }
                }
            }
            if (i + npbuf < cnt_w) {
                fence_proxy_async_smem();  // this lane's reads/writes of the buffer
                __syncwarp();              // before its next tensor copy
                const int v = issue(i + npbuf);
                if (k) vbuf1 = v; else vbuf0 = v;
            }
            if (ABSP_PAGE_PREFETCH > 0) prefetch(i + 1 + ABSP_PAGE_PREFETCH);
        }
        stampk(p.stamp_slot, 7);                 // warp 0 attended its pages
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l8 += __shfl_xor_sync(0xffffffffu, l8, 1);
        l8 += __shfl_xor_sync(0xffffffffu, l8, 2);
        if (!any0) {
            m0 = -INFINITY;
            m8 = -INFINITY;
        }

        // ------------------------------------------- E: merge partials --
        // Warps merge in shared memory into this CTA's partial (O, M, L);
        // with C > 1 CTA r owns output channels [r * 128/C, (r + 1) * 128/C)
        // of every row, receives that slice of every CTA's partial (16-byte
        // asynchronous stores counted on its mbarrier, its own included),
        // merges the C partials and writes the slice.
        // Warp partials: with G <= 8 each warp writes its partial (O rows,
        // then (M, L) pairs) into its own page buffers, which only it used,
        // so no block barrier is needed first; a wider group's partials
        // span the page buffers of several warps and wait for all of them.
        constexpr int kWarpStride = NPB * kPageSmem / 4;   // floats
        float* Ow = reinterpret_cast<float*>(regB);
        auto ow_at = [&](int w, int row) -> float* {
            return BIG_GROUP ? Ow + (w * G + row) * kD : Ow + w * kWarpStride + row * kD;
        };
        auto ml_at = [&](int w, int row) -> float* {
            return BIG_GROUP ? Ow + kWarps * G * kD + (w * G + row) * 2
                             : Ow + w * kWarpStride + G * kD + row * 2;
        };
        if constexpr (BIG_GROUP) {
            __syncthreads();                               // page buffers are dead
        } else {
            __syncwarp();                                  // this warp's reads of them are done
        }
        if (g < G) {
            float* orow = ow_at(warp, g);
#pragma unroll
            for (int t = 0; t < 16; ++t)
                *reinterpret_cast<float2*>(&orow[t * 8 + 2 * t4]) = make_float2(o[t][0], o[t][1]);
            if (t4 == 0) *reinterpret_cast<float2*>(ml_at(warp, g)) = make_float2(m0, l0);
        }
        if constexpr (BIG_GROUP) {
            if (g + 8 < G) {
                float* orow = ow_at(warp, g + 8);
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    *reinterpret_cast<float2*>(&orow[t * 8 + 2 * t4]) = make_float2(o[t][2], o[t][3]);
                if (t4 == 0) *reinterpret_cast<float2*>(ml_at(warp, g + 8)) = make_float2(m8, l8);
            }
        }
        __syncthreads();
        stampk(p.stamp_slot, 8);                 // warp partials in shared memory
        if constexpr ((MODE & kModeSelect) == 0) cluster_wait();  // B0
        __nv_bfloat16* outp = p.out + (static_cast<int64_t>(s) * p.kv.Hq + h * G) * kD;
        // this CTA's partial of 4 channels of one row, with the row's M and
        // L: the weights exp2(m_w - M) of the warp partials are computed in
        // place by every thread of the row (a row with no valid token has
        // M = -inf and gets zero weights)
        auto cta_partial = [&](int row, int d, float& M, float& L) -> float4 {
            float2 mv[kWarps];
            M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                mv[w] = *reinterpret_cast<const float2*>(ml_at(w, row));
                M = fmaxf(M, mv[w].x);
            }
            L = 0.0f;
            float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float e = M != -INFINITY ? fast_exp2(mv[w].x - M) : 0.0f;
                L = fmaf(mv[w].y, e, L);
                const float4 v = *reinterpret_cast<const float4*>(ow_at(w, row) + d);
                a.x = fmaf(v.x, e, a.x);
                a.y = fmaf(v.y, e, a.y);
                a.z = fmaf(v.z, e, a.z);
                a.w = fmaf(v.w, e, a.w);
            }
            return a;
        };
        if (C == 1) {
#pragma unroll 1
            for (int idx = tid; idx < G * (kD / 4); idx += kThreads) {
                const int row = idx / (kD / 4), d = (idx % (kD / 4)) * 4;
                float M, L;
                const float4 a = cta_partial(row, d, M, L);
                const float r = L > 0.0f ? fast_rcp(L) : 0.0f;
                // 4-byte stores: the output is only 4-byte aligned
                uint32_t* o2 = reinterpret_cast<uint32_t*>(outp + row * kD + d);
                o2[0] = pack_bf16x2(a.x * r, a.y * r);
                o2[1] = pack_bf16x2(a.z * r, a.w * r);
            }
            return;
        }
        const int ds = kD >> lgC;                           // channels per slice, >= 8
        const int lgds = 7 - lgC;
        float* recvO = reinterpret_cast<float*>(regA);      // [C][G][ds]
        float* recvML = recvO + C * G * ds;                 // [C][G][2]: (M, L)
        const uint32_t bar_merge = smem_u32(&sm.bar_merge);
#pragma unroll 1
        for (int idx = tid; idx < G * (kD / 4); idx += kThreads) {
            const int row = idx / (kD / 4), d4 = idx % (kD / 4), d = d4 * 4;
            float M, L;
            const float4 a = cta_partial(row, d, M, L);
            const uint32_t owner = static_cast<uint32_t>(d >> lgds);
            float* dst = &recvO[(rank * G + row) * ds + (d - static_cast<int>(owner) * ds)];
            // to every owner by st.async, this CTA included, so that the
            // owner's mbarrier covers its own slice too (no block barrier)
            st_async_v4(dsmem_addr(smem_u32(dst), owner), a.x, a.y, a.z, a.w,
                        dsmem_addr(bar_merge, owner));
            if (d4 < static_cast<int>(C)) {   // the row's (M, L) to owner d4
                const uint32_t o = static_cast<uint32_t>(d4);
                float* ml = &recvML[(rank * G + row) * 2];
                st_async_v2(dsmem_addr(smem_u32(ml), o), M, L, dsmem_addr(bar_merge, o));
            }
        }
        // every CTA's slice of its partial has arrived (each sends only
        // after its own page lookups, so no CTA leaves while another may
        // still read its staged page ids)
        mbar_wait_bounded<true>(bar_merge, 0, p.err, 3, kWaitNs);
        stampk(p.stamp_slot, 9);                 // every CTA's partial slice here
        // two channels of one row per 4 consecutive lanes, each lane taking
        // every 4th partial: the row's M and L and the weighted sums are
        // reduced over the 4 lanes by 2-step shuffles (no block barrier
        // between the weights and the sums)
        const int tot = G * ds * 2;
        for (int base = 0; base < tot; base += kThreads) {
            if (base + (tid & ~31) >= tot) break;     // whole warps (full-mask shuffles)
            const int idx = base + tid;
            const bool act = idx < tot;
            const int pr = act ? idx >> 2 : 0, qtr = idx & 3;
            const int row = pr >> (lgds - 1), dl = (pr & (ds / 2 - 1)) * 2;
            float2 ml[4];
            float M = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = 4 * j + qtr;
                ml[j] = act && r < static_cast<int>(C)
                            ? *reinterpret_cast<const float2*>(&recvML[(r * G + row) * 2])
                            : make_float2(-INFINITY, 0.0f);
                M = fmaxf(M, ml[j].x);
            }
            M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
            M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
            float L = 0.0f, a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = 4 * j + qtr;
                if (act && r < static_cast<int>(C)) {
                    const float e = M != -INFINITY ? fast_exp2(ml[j].x - M) : 0.0f;
                    L = fmaf(ml[j].y, e, L);
                    const float2 v =
                        *reinterpret_cast<const float2*>(&recvO[(r * G + row) * ds + dl]);
                    a0 = fmaf(v.x, e, a0);
                    a1 = fmaf(v.y, e, a1);
                }
            }
            L += __shfl_xor_sync(0xffffffffu, L, 1);
            a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
            a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
            L += __shfl_xor_sync(0xffffffffu, L, 2);
            a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
            a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
            const float rl = L > 0.0f ? fast_rcp(L) : 0.0f;
            a0 *= rl;
            a1 *= rl;
            if (act && qtr == 0)
                *reinterpret_cast<uint32_t*>(outp + row * kD + rank * ds + dl) = pack_bf16x2(a0, a1);
        }
#ifdef ABSP_PHASE_STAMPS
        __syncthreads();
#endif
        stampk(p.stamp_slot, 10);                // output slice written
    }
}

constexpr int kCacheDevices = 16;  // devices with cached launch state

// the last 8 (cluster size, shared bytes) shapes asked about on one device
struct ShapeCache {
    int c[8] = {};
    size_t smem[8] = {};
    int fit[8] = {};
    int next = 0;
    int find(int C, size_t bytes) const {
        for (int i = 0; i < 8; ++i)
            if (c[i] == C && smem[i] == bytes) return fit[i];
        return -1;
    }
    void insert(int C, size_t bytes, int f) {
        c[next] = C;
        smem[next] = bytes;
        fit[next] = f;
        next = (next + 1) & 7;
    }
};

template <int MODE, bool BIG, bool EARLY, bool BF16C, bool GM, bool DIAG = false, int NPB = 1>
cudaError_t launch_mode(const Params& prm, size_t smem, int C, int pairs, bool pdl,
                        const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t st,
                        bool* fits) {
    auto kern = decode_kernel<MODE, BIG, EARLY, BF16C, GM, DIAG, NPB>;
    // per device (function attributes belong to a device's context) and
    // per shape: whether one cluster of C CTAs with `smem` bytes fits
    static std::mutex mu;
    static bool configured[kCacheDevices] = {};
    static ShapeCache shapes[kCacheDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cached = dev >= 0 && dev < kCacheDevices;
    int fit = -1;
    // the one-time set-up below may run while the caller captures `st` into
    // a graph: relaxed capture mode lets these calls (which touch no stream)
    // through without disturbing the capture
    cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
    cudaThreadExchangeStreamCaptureMode(&mode);
    struct RestoreMode {
        cudaStreamCaptureMode* m;
        ~RestoreMode() { cudaThreadExchangeStreamCaptureMode(m); }
    } restore{&mode};
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!cached || !configured[dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     227 * 1024);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            if (cached) configured[dev] = true;
        }
        if (cached) fit = shapes[dev].find(C, smem);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pairs * C);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (fit < 0) {
        // can one cluster of this shape be resident?  A failed query is not
        // an answer: it is not cached and the launch below reports the error
        std::lock_guard<std::mutex> lock(mu);
        int nclusters = 0;
        cudaLaunchConfig_t q = cfg;   // the query needs no stream
        q.stream = nullptr;
        if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &q) == cudaSuccess) {
            fit = nclusters > 0 ? 1 : 0;
            if (cached) shapes[dev].insert(C, smem, fit);
        } else {
            cudaGetLastError();
            fit = 1;
        }
    }
    *fits = fit != 0;
    if (!fit) return cudaSuccess;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, prm, *tmk, *tmv);
}

}  // namespace

#ifndef ABSP_DECODE_CTAS_PER_SM
#define ABSP_DECODE_CTAS_PER_SM 2   // CTA count the cluster size aims for, per SM
#endif

#ifndef ABSP_DECODE_ROWS_PER_CTA
#define ABSP_DECODE_ROWS_PER_CTA 256  // score rows per CTA the cluster size aims for
#endif
#ifndef ABSP_DECODE_PAGES_PER_CTA
#define ABSP_DECODE_PAGES_PER_CTA 16  // selected pages per CTA (two per warp)
#endif

// Cluster size: enough CTAs to cover the SMs about ABSP_DECODE_CTAS_PER_SM
// times, at most 16, and no more than it takes to give each CTA about
// ABSP_DECODE_ROWS_PER_CTA of the largest head's score rows (nmax blocks)
// and about ABSP_DECODE_PAGES_PER_CTA of a head's selected pages (budget /
// 16).  Past that point more CTAs per head add cluster-wide waits and
// merge partials but take little work off the chain: measured on the
// Llama-shaped 32K layers (up to 2048 blocks, 128 selected pages per head),
// 8 CTAs per head beat 16 at batch 1 (10.36 vs 10.46 us per layer-step) and
// halve the time per launch of independent launches that overlap (3.5 vs
// 6.9 us), while 4 CTAs (four pages per warp) took 13.7 us; on the 128K
// layer (8192 blocks, 256 pages) 16 beat 8 (18.0 vs 19.6 us).
// With the throughput hint the work per CTA doubles (half the CTAs).
static int pick_cluster(int pairs, int num_sms, int nmax, int budget, bool throughput) {
    const int rows = ABSP_DECODE_ROWS_PER_CTA << (throughput ? 1 : 0);
    const int pages = ABSP_DECODE_PAGES_PER_CTA << (throughput ? 1 : 0);
    const int need = std::max((nmax + rows - 1) / rows, (budget / kPage + pages - 1) / pages);
    int C = 1;
    while (C < 16 && pairs * C * 2 <= ABSP_DECODE_CTAS_PER_SM * num_sms && C < need) C *= 2;
    return C;
}

// centroid format x score aggregation: each pair is its own kernel, so the
// default one (INT4, sum) carries no code of the others
template <int MODE, bool BIG, bool EARLY>
cudaError_t launch_variant(bool bf, bool gm, const Params& prm, size_t smem, int C, int pairs,
                           bool pdl, const CUtensorMap* tmk, const CUtensorMap* tmv,
                           cudaStream_t st, bool* fits) {
    if (bf)
        return gm ? launch_mode<MODE, BIG, EARLY, true, true>(prm, smem, C, pairs, pdl, tmk, tmv, st, fits)
                  : launch_mode<MODE, BIG, EARLY, true, false>(prm, smem, C, pairs, pdl, tmk, tmv, st, fits);
    return gm ? launch_mode<MODE, BIG, EARLY, false, true>(prm, smem, C, pairs, pdl, tmk, tmv, st, fits)
              : launch_mode<MODE, BIG, EARLY, false, false>(prm, smem, C, pairs, pdl, tmk, tmv, st, fits);
}

cudaError_t launch_decode(int mode, const DecodeArgs& a, const CUtensorMap* tmk,
                          const CUtensorMap* tmv, bool pdl, bool early_prefetch, cudaStream_t st) {
    static std::atomic<int> sms_of[kCacheDevices];  // SM count per device, 0 = unknown
    int dev = 0, num_sms = 0;
    cudaGetDevice(&dev);
    const bool cached = dev >= 0 && dev < kCacheDevices;
    if (cached) num_sms = sms_of[dev].load(std::memory_order_relaxed);
    if (num_sms <= 0) {
        if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            num_sms <= 0)
            num_sms = 148;
        if (cached) sms_of[dev].store(num_sms, std::memory_order_relaxed);
    }
    const int pairs = a.kv.S * a.kv.Hkv;
    const int G = a.kv.G;
    const bool big = G > 8;
    const bool do_select = (mode & kModeSelect) != 0;
    const bool do_attend = (mode & kModeAttend) != 0;

    Params prm;
    prm.kv = a.kv;
    prm.codes = a.codes;
    prm.scale = a.scale;
    prm.zp = a.zp;
    prm.q = a.q;
    prm.out = a.out;
    prm.sel = a.sel;
    prm.sel_count = a.sel_count;
    prm.kmax = a.kmax;
    prm.budget = a.budget;
    prm.err = a.err;
    prm.qk_scale_log2 = kLog2e / sqrtf(static_cast<float>(kD));
    prm.wg_off = 0;
#ifdef ABSP_PHASE_STAMPS
    prm.stamp_slot = mode == kModeFull ? (g_stamp_launches++ & 63) : -1;
#else
    prm.stamp_slot = -1;
#endif

    int C = pick_cluster(pairs, num_sms, a.nmax, a.budget, a.throughput != 0);
    cudaError_t e = cudaSuccess;
    for (; C >= 1; C /= 2) {
        // region B: scores + select scratch + the code ring, then this CTA's
        // page buffers, then the warp merge; region A: the cluster merge's
        // receive buffers
        size_t regB = 0, regA = 0, scratch = 0, ring = 0;
        if (do_select) {
            // score slots for every row, rounded up to whole groups of 4
            scratch = (static_cast<size_t>(a.nmax + 3) / 4) * 16;
            prm.wg_off = static_cast<uint32_t>(scratch + kSelectScratch);
            const size_t used = scratch + kSelectScratch +
                                (a.group_max ? static_cast<size_t>(G) * kWgStride * 4 : 0);
            ring = (used + 127) & ~static_cast<size_t>(127);
            regB = std::max(regB, ring + static_cast<size_t>(kStages) * kStageBytes);
        }
        // Page buffers per warp: a second one overlaps a page's copy with the
        // previous page's attention but takes the shared memory of a second
        // CTA per SM.  The default fused step (INT4, sum, GQA <= 8, no
        // throughput hint) has its own kernel instance with two, used when
        // the launch's CTAs fit on half the SMs, so that one CTA per SM
        // still leaves room for the next launch; every other instance keeps
        // one (measured: the batch-1 Llama-shaped layer-step 10.37 -> 10.12
        // us; with the extra buffer logic in every instance the batched
        // workloads lost 1 %).
        prm.npbuf = mode == kModeFull && !big && a.cfmt != ABSP_CENTROIDS_BF16 &&
                            !a.group_max && !a.diag_timeout && !a.throughput &&
                            pairs * C * 2 <= num_sms
                        ? 2
                        : 1;
        if (do_attend) {
            regB = std::max(regB, static_cast<size_t>(kWarps) * prm.npbuf * kPageSmem);
            regB = std::max(regB, static_cast<size_t>(kWarps) * G * (kD + 2) * 4);
            // the slice merge's receive buffers: C partial slices of G x
            // 128/C channels and (M, L) per row
            if (C > 1)
                regA = std::max(regA, static_cast<size_t>(G) * kD * 4 + static_cast<size_t>(8) * C * G);
        }
        regB = (regB + 1023) & ~static_cast<size_t>(1023);
        regA = (regA + 127) & ~static_cast<size_t>(127);
        // as many ring stages as region B holds past the select scratch
        prm.nstages = kStages;
        prm.ring_off = static_cast<uint32_t>(ring);
        if (do_select)
            prm.nstages = static_cast<int>(
                std::min<size_t>(kMaxStages, std::max<size_t>(kStages, (regB - ring) / kStageBytes)));
        prm.scratch_off = static_cast<uint32_t>(scratch);
        prm.regA_off = static_cast<uint32_t>(regB);
        prm.small_off = static_cast<uint32_t>(regB + regA);
        prm.qs_off = static_cast<uint32_t>(regB + regA + ((sizeof(Small) + 15) & ~static_cast<size_t>(15)));
        // the fused step stages whole page-table rows in what is left of a
        // two-CTAs-per-SM share of shared memory (rows that do not fit use
        // the per-CTA slices or global reads)
        const size_t tail = (static_cast<size_t>(prm.qs_off) + static_cast<size_t>(G) * kD * 2 +
                             static_cast<size_t>(a.kmax) * 4 + 15) & ~static_cast<size_t>(15);
        prm.ptrow_off = static_cast<uint32_t>(tail);
        prm.pt_cap = 0;
        const size_t share = prm.npbuf == 2 ? 224 * 1024 : 112 * 1024;  // per-CTA budget
        if (do_select && do_attend && 1024 + tail < share)
            prm.pt_cap = static_cast<int32_t>(
                std::min<size_t>(a.kv.max_pages, (share - 1024 - tail) / 4) & ~static_cast<size_t>(3));
        const size_t smem = 1024 + tail + static_cast<size_t>(prm.pt_cap) * 4;
        if (smem > 227 * 1024) return cudaErrorInvalidValue;
        bool fits = false;
        const bool early = early_prefetch && mode == kModeFull;
        const bool bf = a.cfmt == ABSP_CENTROIDS_BF16, gm = a.group_max != 0;
        if (a.diag_timeout) {
            // the failure-path diagnostic: INT4 centroids, sum aggregation,
            // GQA group <= 8, no early prefetch (checked by the caller)
            e = mode == kModeSelect
                    ? launch_mode<kModeSelect, false, false, false, false, true>(
                          prm, smem, C, pairs, pdl, tmk, tmv, st, &fits)
                    : launch_mode<kModeFull, false, false, false, false, true>(
                          prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
        } else if (mode == kModeAttend) {
            e = big ? launch_mode<kModeAttend, true, false, false, false>(
                          prm, smem, C, pairs, pdl, tmk, tmv, st, &fits)
                    : launch_mode<kModeAttend, false, false, false, false>(
                          prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
        } else if (mode == kModeSelect) {
            e = big ? launch_variant<kModeSelect, true, false>(bf, gm, prm, smem, C, pairs, pdl,
                                                               tmk, tmv, st, &fits)
                    : launch_variant<kModeSelect, false, false>(bf, gm, prm, smem, C, pairs, pdl,
                                                                tmk, tmv, st, &fits);
        } else if (big) {
            e = early ? launch_variant<kModeFull, true, true>(bf, gm, prm, smem, C, pairs, pdl,
                                                              tmk, tmv, st, &fits)
                      : launch_variant<kModeFull, true, false>(bf, gm, prm, smem, C, pairs, pdl,
                                                               tmk, tmv, st, &fits);
        } else if (prm.npbuf == 2) {
            e = early ? launch_mode<kModeFull, false, true, false, false, false, 2>(
                            prm, smem, C, pairs, pdl, tmk, tmv, st, &fits)
                      : launch_mode<kModeFull, false, false, false, false, false, 2>(
                            prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
        } else {
            e = early ? launch_variant<kModeFull, false, true>(bf, gm, prm, smem, C, pairs, pdl,
                                                               tmk, tmv, st, &fits)
                      : launch_variant<kModeFull, false, false>(bf, gm, prm, smem, C, pairs, pdl,
                                                                tmk, tmv, st, &fits);
        }
        if (e != cudaSuccess || fits) return e;
        // this cluster shape cannot be resident: retry with a smaller one
    }
    e = cudaErrorInvalidClusterSize;
    return e;
}

}  // namespace absp

#ifdef ABSP_PHASE_STAMPS
// Profiling build only: restart the slot count; copy the stamps (globaltimer
// ns, then clock64 ticks, each [64][160][24]) to host memory.
extern "C" __attribute__((visibility("default"))) void absp_phase_stamps_reset() {
    absp::g_stamp_launches = 0;
}
extern "C" __attribute__((visibility("default"))) int absp_phase_stamps_copy(void* t, void* c) {
    cudaError_t e = cudaMemcpyFromSymbol(t, absp::g_stamp_t, sizeof(absp::g_stamp_t));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(c, absp::g_stamp_c, sizeof(absp::g_stamp_c));
    return static_cast<int>(e);
}
#endif
