// Steps 3-5 of AB-Sparse (arXiv 2605.12110), Fig. 1: query-centroid dot
// product estimation over INT4 centroid codes, per-head top-K block
// selection under a token budget (Fig. 9), and exact softmax attention over
// the selected blocks' tokens gathered from the paged cache.
//
// One thread-block cluster of C CTAs (C in 1..16) handles one
// (sequence, KV head).  Phases of decode_kernel:
//   A  score:   CTA r streams its contiguous 1/C share of the head's code
//               rows into shared memory with 1-D bulk copies, scores every
//               row (8 lanes per 64-byte row, 16 codes per lane, fp32) and
//               broadcasts each score into the score array of every CTA of
//               the cluster through distributed shared memory.
//   B  cluster barrier: every CTA now holds all n_h scores.
//   C  select:  every CTA runs the same deterministic radix select (four
//               8-bit digit passes over order-preserving uint32 keys, ties to
//               the lower block index) and an ordered compaction, so all
//               CTAs hold the same ascending block list without another
//               exchange.
//   D  attend:  the selected blocks expand to bs/16 pages each; CTA r takes
//               a contiguous 1/C share of those pages and loads each
//               (page, head) K and V slice with 2-D tensor copies (128-byte
//               swizzle, no multicast).  Each warp owns one page per round:
//               S^T = Q K^T and O += P V on mma.sync bf16 tiles with the GQA
//               group as the 16-row M dimension, online softmax in fp32.
//   E  merge:   warps merge in shared memory; CTAs merge their (m, l, O)
//               partials into CTA 0 through distributed shared memory; CTA 0
//               writes the bf16 output.
// Modes: select only (writes sel / sel_count), attend only (reads them) and
// full (A-E in one launch, the selection never leaves the chip).
#include <algorithm>
#include <cfloat>

#include "absp_internal.cuh"

namespace absp {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStageRows = 256;                    // code rows per bulk stage
constexpr int kStages = 2;
constexpr int kStageBytes = kStageRows * kRowBytes;  // 16 KiB
constexpr int kPagesPerRound = kWarps;             // one page per warp
constexpr int kPageSmem = 4 * 2048;                // K lo/hi, V lo/hi halves
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
};

struct Small {                    // fixed-size shared scratch
    unsigned long long bar[4];    // code stage 0/1, attention, spare
    uint32_t hist[256];
    int32_t misc[32];
    float w[kD];                  // qbar[ch] * scale[ch]
    float zb[kD];                 // 2^23 + zp[ch]
    int4 pinfo[kPagesPerRound];   // {phys, valid, -, -}
    uint32_t scan[kWarps];
};

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) {
    return *reinterpret_cast<const uint32_t*>(p);
}

// Block-wide exclusive prefix sum of one uint32 per thread.
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
    uint32_t base = 0;
    for (int w = 0; w < warp; ++w) base += scan[w];
    __syncthreads();
    return base + inc - v;
}

// Top-k of keys[0..n) (largest keys, ties to the lower index), written to
// out[0..k) in ascending index order.  Requires n <= 65535.
__device__ void block_topk(const uint32_t* keys, int n, int k, int32_t* out, Small& sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k >= n) {
        for (int i = tid; i < n; i += kThreads) out[i] = i;
        __syncthreads();
        return;
    }
    uint32_t prefix = 0, mask = 0;
    int rem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        sm.hist[tid] = 0;  // kThreads == 256 bins
        __syncthreads();
        for (int i = tid; i < n; i += kThreads) {
            const uint32_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 0xFFu], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l scans digits 255-8l down to 248-8l
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = sm.hist[255 - 8 * lane - j];
                tot += c[j];
            }
            uint32_t inc = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += t;
            }
            const uint32_t exc = inc - tot;
            if (exc < static_cast<uint32_t>(rem) && static_cast<uint32_t>(rem) <= inc) {
                uint32_t cum = exc;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (cum + c[j] >= static_cast<uint32_t>(rem)) {
                        sm.misc[0] = 255 - 8 * lane - j;
                        sm.misc[1] = rem - static_cast<int>(cum);
                        break;
                    }
                    cum += c[j];
                }
            }
        }
        __syncthreads();
        prefix |= static_cast<uint32_t>(sm.misc[0]) << shift;
        mask |= 0xFFu << shift;
        rem = sm.misc[1];
        __syncthreads();
    }
    // keys > T are in; of the keys == T the `rem` lowest indices are in.
    const uint32_t T = prefix;
    const int per = (n + kThreads - 1) / kThreads;
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    uint32_t gt = 0, eq = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t key = keys[i];
        gt += key > T;
        eq += key == T;
    }
    const uint32_t ex = block_excl_scan((gt << 16) | eq, sm.scan);
    uint32_t gtb = ex >> 16, eqb = ex & 0xFFFFu;
    const uint32_t r = static_cast<uint32_t>(rem);
    for (int i = i0; i < i1; ++i) {
        const uint32_t key = keys[i];
        if (key > T) {
            out[gtb + min(eqb, r)] = i;
            ++gtb;
        } else if (key == T) {
            if (eqb < r) out[gtb + eqb] = i;
            ++eqb;
        }
    }
    __syncthreads();
}

template <int MODE, bool BIG_GROUP>
__global__ void __launch_bounds__(kThreads, BIG_GROUP ? 1 : 2)
    decode_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* regB = base;                        // scores / pages / warp merge
    uint8_t* regA = base + p.regA_off;           // code ring / cluster merge
    Small& sm = *reinterpret_cast<Small*>(base + p.small_off);
    int32_t* sel_s = reinterpret_cast<int32_t*>(base + p.small_off + sizeof(Small));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t C = cluster_nctarank();
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x / C;
    const int Hkv = p.kv.Hkv, G = p.kv.G;
    const int s = pair / Hkv, h = pair % Hkv;
    const uint32_t bar_code0 = smem_u32(&sm.bar[0]);
    const uint32_t bar_attn = smem_u32(&sm.bar[2]);

    // B0 arrive: matched by the wait before the first remote access.
    cluster_arrive_relaxed();
    if (tid == 0) {
        mbar_init(bar_code0, 1);
        mbar_init(bar_code0 + 8, 1);
        mbar_init(bar_attn, 1);
        fence_mbar_init();
    }
    // Nothing in global memory is read before this point.
    pdl_wait();
    pdl_trigger();
    __syncthreads();

    int len = p.kv.seq_lens[s];
    if (len < 0 || len > p.kv.max_pages * kPage) {
        if (tid == 0 && rank == 0 && h == 0) set_error(p.err, ABSP_ERR_DEVICE_FAULT, s);
        len = 0;
    }
    const int bs = p.kv.bs[h];
    const int spb = bs / kPage;
    const int n = (len + bs - 1) / bs;
    int K = 0;

    if constexpr ((MODE & kModeSelect) != 0) {
        // ---------------------------------------------------- A: score --
        K = min(n, max(1, p.budget / bs));
        const int per = (n + static_cast<int>(C) - 1) / static_cast<int>(C);
        const int r0 = min(n, static_cast<int>(rank) * per);
        const int nrows = min(n, r0 + per) - r0;
        const int nchunks = (nrows + kStageRows - 1) / kStageRows;
        const uint8_t* cbase =
            p.codes + (static_cast<int64_t>(s) * p.kv.rows_per_seq + p.kv.row_base[h] + r0) * kRowBytes;
        if (tid == 0) {
            for (int c = 0; c < min(nchunks, kStages); ++c) {
                const int rows = min(kStageRows, nrows - c * kStageRows);
                mbar_arrive_expect_tx(bar_code0 + 8 * c, rows * kRowBytes);
                bulk_g2s(smem_u32(regA + c * kStageBytes), cbase + c * kStageBytes,
                         rows * kRowBytes, bar_code0 + 8 * c);
            }
        }
        if (tid < kD) {
            const __nv_bfloat16* qh = p.q + (static_cast<int64_t>(s) * p.kv.Hq + h * G) * kD + tid;
            float qb = 0.0f;
            for (int j = 0; j < G; ++j) qb += __bfloat162float(qh[j * kD]);
            const int64_t pi = (static_cast<int64_t>(s) * Hkv + h) * kD + tid;
            sm.w[tid] = qb * p.scale[pi];
            sm.zb[tid] = 8388608.0f + static_cast<float>(p.zp[pi]);
        }
        __syncthreads();
        const int sub = tid & 7, grp = tid >> 3;  // 32 groups of 8 lanes
        float wr[16], zr[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            wr[k] = sm.w[sub * 16 + k];
            zr[k] = sm.zb[sub * 16 + k];
        }
        float* scores = reinterpret_cast<float*>(regB);
        const uint32_t scores_u32 = smem_u32(scores);
        cluster_wait();  // B0: every CTA of the cluster is running
        for (int c = 0; c < nchunks; ++c) {
            const int stage = c % kStages;
            mbar_wait_bounded(bar_code0 + 8 * stage, (c / kStages) & 1, p.err, 1);
            const int rows = min(kStageRows, nrows - c * kStageRows);
            const uint8_t* sbuf = regA + stage * kStageBytes;
            for (int rb = 0; rb < rows; rb += kThreads / 8) {
                const int r = rb + grp;
                const bool ok = r < rows;
                uint2 x = make_uint2(0u, 0u);
                if (ok) x = *reinterpret_cast<const uint2*>(sbuf + r * kRowBytes + sub * 8);
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float f = __uint_as_float(0x4B000000u | ((x.x >> (4 * k)) & 0xFu)) - zr[k];
                    acc = fmaf(wr[k], f, acc);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float f =
                        __uint_as_float(0x4B000000u | ((x.y >> (4 * k)) & 0xFu)) - zr[8 + k];
                    acc = fmaf(wr[8 + k], f, acc);
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                if (ok) {
                    const uint32_t row = static_cast<uint32_t>(r0 + c * kStageRows + r);
                    for (uint32_t dst = sub; dst < C; dst += 8)
                        dsmem_st_f32(dsmem_addr(scores_u32 + 4 * row, dst), acc);
                }
            }
            __syncthreads();
            if (tid == 0 && c + kStages < nchunks) {
                const int cn = c + kStages;
                const int rows_n = min(kStageRows, nrows - cn * kStageRows);
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar_code0 + 8 * stage, rows_n * kRowBytes);
                bulk_g2s(smem_u32(regA + stage * kStageBytes), cbase + cn * kStageBytes,
                         rows_n * kRowBytes, bar_code0 + 8 * stage);
            }
        }
        // ---------------------------------------------- B: all scores in --
        cluster_arrive();
        cluster_wait();
        if (MODE == kModeSelect && rank != 0) return;  // no remote access follows

        // --------------------------------------------------- C: select --
        uint32_t* keys = reinterpret_cast<uint32_t*>(regB);
        for (int i = tid; i < n; i += kThreads) keys[i] = order_key(scores[i]);
        __syncthreads();
        block_topk(keys, n, K, sel_s, sm);
        if (MODE == kModeSelect) {
            int32_t* dst = p.sel + (static_cast<int64_t>(s) * Hkv + h) * p.kmax;
            for (int i = tid; i < K; i += kThreads) dst[i] = sel_s[i];
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
        const int pb = static_cast<int>((static_cast<int64_t>(P) * rank) / C);
        const int pe = static_cast<int>((static_cast<int64_t>(P) * (rank + 1)) / C);
        const int g = lane >> 2, t4 = lane & 3;
        const __nv_bfloat16* qg = p.q + (static_cast<int64_t>(s) * p.kv.Hq + h * G) * kD;
        uint32_t qa0[8], qa2[8], qa1[8], qa3[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            qa0[j] = g < G ? ld_u32(qg + g * kD + 16 * j + 2 * t4) : 0u;
            qa2[j] = g < G ? ld_u32(qg + g * kD + 16 * j + 8 + 2 * t4) : 0u;
            if constexpr (BIG_GROUP) {
                qa1[j] = g + 8 < G ? ld_u32(qg + (g + 8) * kD + 16 * j + 2 * t4) : 0u;
                qa3[j] = g + 8 < G ? ld_u32(qg + (g + 8) * kD + 16 * j + 8 + 2 * t4) : 0u;
            } else {
                qa1[j] = 0u;
                qa3[j] = 0u;
            }
        }
        float o[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
        float m0 = -FLT_MAX, m8 = -FLT_MAX, l0 = 0.0f, l8 = 0.0f;
        bool any0 = false;  // this warp has seen at least one valid token
        const int32_t* pt = p.kv.page_table + static_cast<int64_t>(s) * p.kv.max_pages;
        const float qks = p.qk_scale_log2;
        __syncthreads();  // the score keys in regB are dead from here on

        int round = 0;
        for (int bp = pb; bp < pe; bp += kPagesPerRound, ++round) {
            const int np = min(kPagesPerRound, pe - bp);
            if (tid < np) {
                const int j = bp + tid;
                const int b = sel_s[j / spb];
                int valid = 0, phys = -1;
                if (b >= 0) {
                    const int lp = b * spb + (j % spb);
                    valid = min(kPage, len - lp * kPage);
                    if (valid > 0) {
                        phys = pt[lp];
                        if (phys < 0 || phys >= p.kv.num_phys_pages) {
                            set_error(p.err, ABSP_ERR_DEVICE_FAULT, s);
                            valid = 0;
                        }
                    } else {
                        valid = 0;
                    }
                }
                sm.pinfo[tid] = make_int4(phys, valid, 0, 0);
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t bytes = 0;
                for (int i = 0; i < np; ++i) bytes += sm.pinfo[i].y > 0 ? kPageSmem : 0;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar_attn, bytes);
                for (int i = 0; i < np; ++i) {
                    if (sm.pinfo[i].y <= 0) continue;
                    const int y = (sm.pinfo[i].x * Hkv + h) * kPage;
                    const uint32_t dst = smem_u32(regB + i * kPageSmem);
                    tma_load_2d(dst, &tmk, 0, y, bar_attn);
                    tma_load_2d(dst + 2048, &tmk, 64, y, bar_attn);
                    tma_load_2d(dst + 4096, &tmv, 0, y, bar_attn);
                    tma_load_2d(dst + 6144, &tmv, 64, y, bar_attn);
                }
            }
            mbar_wait_bounded(bar_attn, round & 1, p.err, 2);
            const int valid = warp < np ? sm.pinfo[warp].y : 0;
            if (valid > 0) {
                uint8_t* pg = regB + warp * kPageSmem;
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
                    if constexpr (BIG_GROUP) {
                        mma_bf16(s0[0], s0[1], s0[2], s0[3], qa0[j], qa1[j], qa2[j], qa3[j], b0, b1);
                        mma_bf16(s1[0], s1[1], s1[2], s1[3], qa0[j], qa1[j], qa2[j], qa3[j], b2, b3);
                    } else {
                        mma_bf16_top(s0[0], s0[1], qa0[j], qa2[j], b0, b1);
                        mma_bf16_top(s1[0], s1[1], qa0[j], qa2[j], b2, b3);
                    }
                }
                // scale to log2 units and mask tokens past the end
                const int ta = 2 * t4, tb = 8 + 2 * t4;
                float x0 = ta < valid ? s0[0] * qks : -INFINITY;
                float x1 = ta + 1 < valid ? s0[1] * qks : -INFINITY;
                float x2 = tb < valid ? s1[0] * qks : -INFINITY;
                float x3 = tb + 1 < valid ? s1[1] * qks : -INFINITY;
                float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                // valid >= 1 so token 0 is valid: mx is finite
                const float mn0 = fmaxf(m0, mx);
                const float corr0 = any0 ? exp2f(m0 - mn0) : 0.0f;
                const uint32_t pa0 = pack_bf16x2(exp2f(x0 - mn0), exp2f(x1 - mn0));
                const uint32_t pa2 = pack_bf16x2(exp2f(x2 - mn0), exp2f(x3 - mn0));
                const float ps0 = bf16lo(pa0) + bf16hi(pa0) + bf16lo(pa2) + bf16hi(pa2);
                l0 = l0 * corr0 + ps0;
                m0 = mn0;
                uint32_t pa1 = 0u, pa3 = 0u;
                float corr8 = 1.0f;
                if constexpr (BIG_GROUP) {
                    float y0 = ta < valid ? s0[2] * qks : -INFINITY;
                    float y1 = ta + 1 < valid ? s0[3] * qks : -INFINITY;
                    float y2 = tb < valid ? s1[2] * qks : -INFINITY;
                    float y3 = tb + 1 < valid ? s1[3] * qks : -INFINITY;
                    float my = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
                    my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, 1));
                    my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, 2));
                    const float mn8 = fmaxf(m8, my);
                    corr8 = any0 ? exp2f(m8 - mn8) : 0.0f;
                    pa1 = pack_bf16x2(exp2f(y0 - mn8), exp2f(y1 - mn8));
                    pa3 = pack_bf16x2(exp2f(y2 - mn8), exp2f(y3 - mn8));
                    l8 = l8 * corr8 + bf16lo(pa1) + bf16hi(pa1) + bf16lo(pa3) + bf16hi(pa3);
                    m8 = mn8;
                }
                any0 = true;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    o[i][0] *= corr0;
                    o[i][1] *= corr0;
                    if constexpr (BIG_GROUP) {
                        o[i][2] *= corr8;
                        o[i][3] *= corr8;
                    }
                }
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
            __syncthreads();  // page buffers are reused next round
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l8 += __shfl_xor_sync(0xffffffffu, l8, 1);
        l8 += __shfl_xor_sync(0xffffffffu, l8, 2);
        if (!any0) {
            m0 = -INFINITY;
            m8 = -INFINITY;
        }

        // ------------------------------------------- E: merge partials --
        float* Ow = reinterpret_cast<float*>(regB);       // [warps][G][128]
        float* mw = Ow + kWarps * G * kD;                  // [warps][G]
        float* lw = mw + kWarps * G;
        if (g < G) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                Ow[(warp * G + g) * kD + i * 8 + 2 * t4] = o[i][0];
                Ow[(warp * G + g) * kD + i * 8 + 2 * t4 + 1] = o[i][1];
            }
            if (t4 == 0) {
                mw[warp * G + g] = m0;
                lw[warp * G + g] = l0;
            }
        }
        if constexpr (BIG_GROUP) {
            if (g + 8 < G) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    Ow[(warp * G + g + 8) * kD + i * 8 + 2 * t4] = o[i][2];
                    Ow[(warp * G + g + 8) * kD + i * 8 + 2 * t4 + 1] = o[i][3];
                }
                if (t4 == 0) {
                    mw[warp * G + g + 8] = m8;
                    lw[warp * G + g + 8] = l8;
                }
            }
        }
        __syncthreads();
        if constexpr ((MODE & kModeSelect) == 0) cluster_wait();  // B0
        float* partO = reinterpret_cast<float*>(regA);    // [C][G][128]
        float* partM = partO + C * G * kD;                 // [C][G]
        float* partL = partM + C * G;
        __nv_bfloat16* outp = p.out + (static_cast<int64_t>(s) * p.kv.Hq + h * G) * kD;
        for (int idx = tid; idx < G * kD; idx += kThreads) {
            const int row = idx >> 7, d = idx & (kD - 1);
            float M = -INFINITY;
            for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mw[w * G + row]);
            float L = 0.0f, Oacc = 0.0f;
            if (M != -INFINITY) {
                for (int w = 0; w < kWarps; ++w) {
                    const float f = exp2f(mw[w * G + row] - M);
                    L += lw[w * G + row] * f;
                    Oacc += Ow[(w * G + row) * kD + d] * f;
                }
            }
            if (C == 1) {
                outp[row * kD + d] = __float2bfloat16_rn(L > 0.0f ? Oacc / L : 0.0f);
            } else {
                const uint32_t lo = smem_u32(&partO[(rank * G + row) * kD + d]);
                dsmem_st_f32(dsmem_addr(lo, 0), Oacc);
                if (d == 0) {
                    dsmem_st_f32(dsmem_addr(smem_u32(&partM[rank * G + row]), 0), M);
                    dsmem_st_f32(dsmem_addr(smem_u32(&partL[rank * G + row]), 0), L);
                }
            }
        }
        if (C > 1) {
            cluster_arrive();
            cluster_wait();
            if (rank == 0) {
                for (int idx = tid; idx < G * kD; idx += kThreads) {
                    const int row = idx >> 7, d = idx & (kD - 1);
                    float M = -INFINITY;
                    for (uint32_t r = 0; r < C; ++r) M = fmaxf(M, partM[r * G + row]);
                    float L = 0.0f, Oacc = 0.0f;
                    if (M != -INFINITY) {
                        for (uint32_t r = 0; r < C; ++r) {
                            const float f = exp2f(partM[r * G + row] - M);
                            L += partL[r * G + row] * f;
                            Oacc += partO[(r * G + row) * kD + d] * f;
                        }
                    }
                    outp[row * kD + d] = __float2bfloat16_rn(L > 0.0f ? Oacc / L : 0.0f);
                }
            }
        }
    }
}

template <int MODE, bool BIG>
cudaError_t launch_mode(const Params& prm, size_t smem, int C, int pairs, bool pdl,
                        const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t st,
                        bool* fits) {
    auto kern = decode_kernel<MODE, BIG>;
    static bool configured = false;   // attributes are per function, set once
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             227 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        configured = true;
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
    // can at least one cluster of this shape be resident?  (cached per shape)
    static int cache_c[8] = {0}, cache_fit[8] = {0};
    static size_t cache_smem[8] = {0};
    int fit = -1;
    for (int i = 0; i < 8; ++i)
        if (cache_c[i] == C && cache_smem[i] == smem) fit = cache_fit[i];
    if (fit < 0) {
        int nclusters = 0;
        cudaError_t e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
        if (e != cudaSuccess) {
            cudaGetLastError();
            nclusters = 0;
        }
        fit = nclusters > 0 ? 1 : 0;
        static int next = 0;
        cache_c[next] = C;
        cache_smem[next] = smem;
        cache_fit[next] = fit;
        next = (next + 1) & 7;
    }
    *fits = fit != 0;
    if (!fit) return cudaSuccess;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, prm, *tmk, *tmv);
}

}  // namespace

// Cluster size: enough CTAs to cover the SMs about twice, at most 16.
static int pick_cluster(int pairs, int num_sms) {
    int C = 1;
    while (C < 16 && pairs * C * 2 <= 2 * num_sms) C *= 2;
    return C;
}

cudaError_t launch_decode(int mode, const DecodeArgs& a, const CUtensorMap* tmk,
                          const CUtensorMap* tmv, bool pdl, cudaStream_t st) {
    static int num_sms = 0;
    if (num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (num_sms <= 0) num_sms = 148;
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

    int C = pick_cluster(pairs, num_sms);
    cudaError_t e = cudaSuccess;
    for (; C >= 1; C /= 2) {
        size_t regB = 0, regA = 0;
        if (do_select) {
            regB = std::max(regB, static_cast<size_t>(a.nmax) * 4);
            regA = std::max(regA, static_cast<size_t>(kStages) * kStageBytes);
        }
        if (do_attend) {
            regB = std::max(regB, static_cast<size_t>(kPagesPerRound) * kPageSmem);
            regB = std::max(regB, static_cast<size_t>(kWarps) * G * (kD + 2) * 4);
            if (C > 1) regA = std::max(regA, static_cast<size_t>(C) * G * (kD + 2) * 4);
        }
        regB = (regB + 1023) & ~static_cast<size_t>(1023);
        regA = (regA + 127) & ~static_cast<size_t>(127);
        prm.regA_off = static_cast<uint32_t>(regB);
        prm.small_off = static_cast<uint32_t>(regB + regA);
        const size_t smem = 1024 + regB + regA + sizeof(Small) + static_cast<size_t>(a.kmax) * 4;
        if (smem > 227 * 1024) return cudaErrorInvalidValue;
        bool fits = false;
        switch (mode * 2 + (big ? 1 : 0)) {
            case kModeSelect * 2:
                e = launch_mode<kModeSelect, false>(prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
                break;
            case kModeSelect * 2 + 1:
                e = launch_mode<kModeSelect, true>(prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
                break;
            case kModeAttend * 2:
                e = launch_mode<kModeAttend, false>(prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
                break;
            case kModeAttend * 2 + 1:
                e = launch_mode<kModeAttend, true>(prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
                break;
            case kModeFull * 2:
                e = launch_mode<kModeFull, false>(prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
                break;
            default:
                e = launch_mode<kModeFull, true>(prm, smem, C, pairs, pdl, tmk, tmv, st, &fits);
                break;
        }
        if (e != cudaSuccess || fits) return e;
        // this cluster shape cannot be resident: retry with a smaller one
    }
    e = cudaErrorInvalidClusterSize;
    return e;
}

}  // namespace absp
