// Steps 1-2 of AB-Sparse (arXiv 2605.12110): mean-key block centroids
// (Fig. 1 "block representation"; Fig. 5: centroids are built over all key
// vectors of a head, once) and their INT4 asymmetric per-channel codes
// (Fig. 8).
//
// Kernel shapes.  Both kernels tile a layer by (1024-token chunk, KV head,
// sequence): every CTA covers the same number of tokens whatever the head's
// block size (64, 32 or 16 blocks), so work is balanced across heads.
//   build:    one warp per block; lane L owns channels 4L..4L+3 and reads
//             8 bytes of every key row (a warp reads a full 256-byte row per
//             instruction, coalesced).  Sums are fp64 in token order, so the
//             result is bit-identical to a sequential fp64 mean.  The CTA
//             reduces its per-channel min / max in shared memory and issues
//             one atomic per channel (order-mapped fp64 keys).
//   quantize: reads the fp64 centroids back, derives scale / zero point from
//             the min / max (fp64, IEEE division, rint half-to-even) and
//             writes packed nibbles: lane L writes 2 bytes of each 64-byte
//             row.  The BF16 store (the unquantised precision of Fig. 13)
//             instead writes each centroid rounded to bf16, 256-byte rows.
#include <algorithm>
#include <mutex>

#include "absp_internal.cuh"

namespace absp {

namespace {

constexpr int kChunkTokens = 1024;
constexpr int kBuildWarps = 8;
constexpr int kBuildSmem = (kChunkTokens / 16) * 128 * 8;   // a chunk's fp64 rows

__device__ __forceinline__ unsigned long long ord_f64(double x) {
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ double unord_f64(unsigned long long k) {
    const unsigned long long u = (k >> 63) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
    return __longlong_as_double(static_cast<long long>(u));
}

__device__ __forceinline__ uint2 ld_nc_u2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_nc_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// x / cnt for a block's token count: a power of two (every full block) is
// an exact scaling by its reciprocal; a ragged tail divides.
__device__ __forceinline__ double mean_of(double x, int cnt, double inv_pow2) {
    return (cnt & (cnt - 1)) == 0 ? x * inv_pow2 : x / static_cast<double>(cnt);
}

// rint(c / sc) (IEEE division, round half to even) without dividing on the
// common path: r = c * inv (inv = 1 / sc rounded) is within 2^-51 |c/sc| of
// the quotient, so unless r lies within 2^-48 max(|r|, 1) of a half-integer
// (where rint could jump) its rint is the quotient's; otherwise divide.
__device__ __forceinline__ double rint_div(double c, double sc, double inv) {
    const double r = c * inv;
    const double fl = floor(r);
    const double d = r - fl;
    if (fabs(d - 0.5) <= fmax(fabs(r), 1.0) * 0x1p-48) return rint(c / sc);
    return d > 0.5 ? fl + 1.0 : fl;
}

// Validated sequence length; faults are recorded once per sequence.
__device__ __forceinline__ int checked_len(const KvDesc& kv, int s, int32_t* err) {
    const int len = kv.seq_lens[s];
    if (len < 0 || len > kv.max_pages * kPage) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
            set_error(err, ABSP_ERR_DEVICE_FAULT, s);
        return -1;
    }
    return len;
}

// fp64 -> bf16, round to nearest even, without double rounding: first round
// to odd into fp32 (truncate, then set the last bit when inexact; fp32 keeps
// 16 more bits than bf16), then round to nearest even into bf16.
__device__ __forceinline__ uint32_t f64_to_bf16_rne(double x) {
    const float f = __double2float_rz(x);
    uint32_t u = __float_as_uint(f);
    if (static_cast<double>(f) != x) u |= 1u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return u >> 16;
}

// Two-pass build: one CTA per (1024-token chunk, KV head, sequence).  Each
// half-warp takes one block at a time; lane l (of 16) owns channels
// 8l .. 8l+7 and reads 16 bytes of every key row (a half-warp reads a whole
// 256-byte row per instruction, a page's 16 rows in flight).  Token-order
// fp64 sums.  The chunk's centroids go to the workspace and to shared
// memory; the CTA's per-channel min / max is taken over the shared copy and
// merged with one atomic per channel into order-mapped keys (the max as the
// key of its negation, so that one fill of ones initialises every key).
__global__ void __launch_bounds__(kBuildWarps * 32)
    centroid_build_kernel(const KvDesc kv, BuildWs w) {
    const int chunk = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x;
    const int hw = tid >> 4, hl = tid & 15;            // half-warp, lane within it
    constexpr int kHalfWarps = kBuildWarps * 2;
    extern __shared__ __align__(16) uint8_t build_smem[];
    auto rows_s = reinterpret_cast<double (*)[kD]>(build_smem);   // [64][128]: a chunk's blocks

    const int len = checked_len(kv, s, w.err);
    const int tok0 = chunk * kChunkTokens;
    if (len <= tok0) return;  // uniform over the CTA

    const int bs = kv.bs[h];
    const int n = (len + bs - 1) / bs;
    const int b_begin = tok0 / bs;
    const int b_end = min(n, (tok0 + kChunkTokens) / bs);
    const int32_t* pt = kv.page_table + static_cast<int64_t>(s) * kv.max_pages;
    double* cent = w.cent + (static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h]) * kD;

    for (int b = b_begin + hw; b < b_end; b += kHalfWarps) {
        const int t0 = b * bs;
        const int cnt = min(bs, len - t0);
        double a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = 0.0;
        for (int tp = t0; tp < t0 + cnt; tp += kPage) {
            const int nt = min(kPage, t0 + cnt - tp);
            const int phys = pt[tp / kPage];
            if (phys < 0 || phys >= kv.num_phys_pages) {
                if (hl == 0) set_error(w.err, ABSP_ERR_DEVICE_FAULT, s);
                continue;
            }
            const __nv_bfloat16* src =
                kv.k_pages + ((static_cast<int64_t>(phys) * kv.Hkv + h) * kPage) * kD + hl * 8;
            uint4 v[kPage];
#pragma unroll
            for (int t = 0; t < kPage; ++t)
                if (t < nt) v[t] = ld_nc_u4(src + t * kD);
#pragma unroll
            for (int t = 0; t < kPage; ++t) {
                if (t < nt) {
                    a[0] += static_cast<double>(bf16lo(v[t].x));
                    a[1] += static_cast<double>(bf16hi(v[t].x));
                    a[2] += static_cast<double>(bf16lo(v[t].y));
                    a[3] += static_cast<double>(bf16hi(v[t].y));
                    a[4] += static_cast<double>(bf16lo(v[t].z));
                    a[5] += static_cast<double>(bf16hi(v[t].z));
                    a[6] += static_cast<double>(bf16lo(v[t].w));
                    a[7] += static_cast<double>(bf16hi(v[t].w));
                }
            }
        }
        // 2^-k for cnt = 2^k (used only then)
        const double dinv = __hiloint2double((1023 - (__ffs(cnt) - 1)) << 20, 0);
        double2* dg = reinterpret_cast<double2*>(cent + static_cast<int64_t>(b) * kD + hl * 8);
        double2* ds = reinterpret_cast<double2*>(&rows_s[b - b_begin][hl * 8]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double2 c = make_double2(mean_of(a[2 * i], cnt, dinv), mean_of(a[2 * i + 1], cnt, dinv));
            dg[i] = c;
            ds[i] = c;
        }
    }
    __syncthreads();
    // per-channel min / max of the chunk's rows: thread t takes channel
    // t % 128 of every other row, the two halves merged by one shuffle-free
    // shared-memory step
    const int nb = b_end - b_begin;
    const int d = tid & (kD - 1), half = tid >> 7;
    double mn = __longlong_as_double(0x7FF0000000000000ll), mx = -mn;
    for (int r = half; r < nb; r += 2) {
        mn = fmin(mn, rows_s[r][d]);
        mx = fmax(mx, rows_s[r][d]);
    }
    __syncthreads();
    double* red = &rows_s[0][0];          // the rows are consumed
    if (half == 1) {
        red[d] = mn;
        red[kD + d] = mx;
    }
    __syncthreads();
    if (half == 0 && nb > 0) {
        mn = fmin(mn, red[d]);
        mx = fmax(mx, red[kD + d]);
        const int64_t pi = (static_cast<int64_t>(s) * kv.Hkv + h) * kD + d;
        const int64_t pairs = static_cast<int64_t>(kv.S) * kv.Hkv * kD;
        atomicMin(w.minmax + pi, ord_f64(mn));
        atomicMin(w.minmax + pairs + pi, ord_f64(-mx));
    }
}

__global__ void __launch_bounds__(kBuildWarps * 32)
    centroid_quantize_kernel(const KvDesc kv, BuildWs w, uint8_t* __restrict__ codes,
                             float* __restrict__ scale_out, int32_t* __restrict__ zp_out) {
    const int chunk = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ double s_scale[kD];
    __shared__ double s_zp[kD];

    const int len = checked_len(kv, s, w.err);
    const int tok0 = chunk * kChunkTokens;
    if (chunk > 0 && len <= tok0) return;  // uniform over the CTA
    const int bs = kv.bs[h];
    const int n = len > 0 ? (len + bs - 1) / bs : 0;

    if (threadIdx.x < kD) {
        const int d = threadIdx.x;
        const int64_t pi = (static_cast<int64_t>(s) * kv.Hkv + h) * kD + d;
        double sc = 0.0, z = 0.0;
        float scf = 0.0f;
        int32_t zi = 0;
        if (n > 0) {
            const int64_t pairs = static_cast<int64_t>(kv.S) * kv.Hkv * kD;
            const double mn = unord_f64(w.minmax[pi]);
            const double mx = -unord_f64(w.minmax[pairs + pi]);
            if (mx > mn) {
                const float f = __double2float_rn((mx - mn) / 15.0);
                if (f > 0.0f) {
                    scf = f;
                    sc = static_cast<double>(f);
                    double zr = rint(-mn / sc);
                    zr = fmin(fmax(zr, -2147483648.0), 2147483647.0);
                    zi = static_cast<int32_t>(zr);
                    z = static_cast<double>(zi);
                }
            }
        }
        s_scale[d] = sc;
        s_zp[d] = z;
        if (chunk == 0) {
            scale_out[pi] = scf;
            zp_out[pi] = zi;
        }
    }
    __syncthreads();
    if (len <= tok0) return;

    const int b_begin = tok0 / bs;
    const int b_end = min(n, (tok0 + kChunkTokens) / bs);
    const int64_t row0 = static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h];
    double sc[4], zz[4], iv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sc[i] = s_scale[lane * 4 + i];
        zz[i] = s_zp[lane * 4 + i];
        iv[i] = sc[i] != 0.0 ? 1.0 / sc[i] : 0.0;
    }
    for (int b = b_begin + warp; b < b_end; b += kBuildWarps) {
        const double2* src = reinterpret_cast<const double2*>(w.cent + (row0 + b) * kD + lane * 4);
        const double2 u = src[0], v = src[1];
        const double c[4] = {u.x, u.y, v.x, v.y};
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t code = 0;
            if (sc[i] != 0.0) {
                double qv = rint_div(c[i], sc[i], iv[i]) + zz[i];
                qv = fmin(fmax(qv, 0.0), 15.0);
                code = static_cast<uint32_t>(qv);
            }
            packed |= code << (4 * i);
        }
        *reinterpret_cast<uint16_t*>(codes + (row0 + b) * kRowBytes + lane * 2) =
            static_cast<uint16_t>(packed);
    }
}

// BF16 centroid store: every fp64 centroid rounded to bf16, 256-byte rows.
__global__ void __launch_bounds__(kBuildWarps * 32)
    centroid_bf16_kernel(const KvDesc kv, BuildWs w, uint8_t* __restrict__ rows_out) {
    const int chunk = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int len = checked_len(kv, s, w.err);
    const int tok0 = chunk * kChunkTokens;
    if (len <= tok0) return;  // uniform over the CTA
    const int bs = kv.bs[h];
    const int n = (len + bs - 1) / bs;
    const int b_begin = tok0 / bs;
    const int b_end = min(n, (tok0 + kChunkTokens) / bs);
    const int64_t row0 = static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h];
    for (int b = b_begin + warp; b < b_end; b += kBuildWarps) {
        const double2* src = reinterpret_cast<const double2*>(w.cent + (row0 + b) * kD + lane * 4);
        const double2 u = src[0], v = src[1];
        uint2 o;
        o.x = f64_to_bf16_rne(u.x) | (f64_to_bf16_rne(u.y) << 16);
        o.y = f64_to_bf16_rne(v.x) | (f64_to_bf16_rne(v.y) << 16);
        *reinterpret_cast<uint2*>(rows_out + (row0 + b) * (2 * kD) + lane * 8) = o;
    }
}

// Incremental update after tokens were appended: one warp per
// (sequence, KV head) recomputes the centroid of the block that holds the
// last token (token-order fp64 sum over that block's keys) and stores it
// under the existing per-channel parameters (INT4, clamped) or as bf16.
// exceeded[s][h] counts INT4 channels whose unclamped code left 0..15.
__global__ void __launch_bounds__(kBuildWarps * 32)
    centroid_append_kernel(const KvDesc kv, uint8_t* __restrict__ codes,
                           const float* __restrict__ scale, const int32_t* __restrict__ zp,
                           int format, int32_t* __restrict__ exceeded, int32_t* err) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.x * kBuildWarps + warp;
    if (pair >= kv.S * kv.Hkv) return;
    const int s = pair / kv.Hkv, h = pair % kv.Hkv;
    int len = kv.seq_lens[s];
    if (len < 0 || len > kv.max_pages * kPage) {
        if (lane == 0 && h == 0) set_error(err, ABSP_ERR_DEVICE_FAULT, s);
        len = 0;
    }
    int count = 0;
    if (len > 0) {
        const int bs = kv.bs[h];
        const int b = (len - 1) / bs;
        const int t0 = b * bs;
        const int32_t* pt = kv.page_table + static_cast<int64_t>(s) * kv.max_pages;
        // page ids of the block first (at most 4), then each page's rows
        // with 16 loads in flight, summed in token order
        int phys[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) phys[i] = t0 + i * kPage < len ? pt[t0 / kPage + i] : 0;
        double a[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int tp = t0 + i * kPage;
            if (tp >= len) break;
            const int nt = min(kPage, len - tp);
            if (phys[i] < 0 || phys[i] >= kv.num_phys_pages) {
                if (lane == 0) set_error(err, ABSP_ERR_DEVICE_FAULT, s);
                continue;
            }
            const __nv_bfloat16* src =
                kv.k_pages + ((static_cast<int64_t>(phys[i]) * kv.Hkv + h) * kPage) * kD + lane * 4;
            uint2 v[kPage];
#pragma unroll
            for (int t = 0; t < kPage; ++t)
                if (t < nt) v[t] = ld_nc_u2(src + t * kD);
#pragma unroll
            for (int t = 0; t < kPage; ++t) {
                if (t < nt) {
                    a[0] += static_cast<double>(bf16lo(v[t].x));
                    a[1] += static_cast<double>(bf16hi(v[t].x));
                    a[2] += static_cast<double>(bf16lo(v[t].y));
                    a[3] += static_cast<double>(bf16hi(v[t].y));
                }
            }
        }
        const double cnt = static_cast<double>(len - t0);
        const int64_t row = static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h] + b;
        if (format == ABSP_CENTROIDS_BF16) {
            uint2 o;
            o.x = f64_to_bf16_rne(a[0] / cnt) | (f64_to_bf16_rne(a[1] / cnt) << 16);
            o.y = f64_to_bf16_rne(a[2] / cnt) | (f64_to_bf16_rne(a[3] / cnt) << 16);
            *reinterpret_cast<uint2*>(codes + row * (2 * kD) + lane * 8) = o;
        } else {
            const int64_t pi = (static_cast<int64_t>(s) * kv.Hkv + h) * kD + lane * 4;
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const double sc = static_cast<double>(scale[pi + i]);
                uint32_t code = 0;
                if (sc > 0.0) {
                    const double qv = rint((a[i] / cnt) / sc) + static_cast<double>(zp[pi + i]);
                    if (qv < 0.0 || qv > 15.0) ++count;
                    code = static_cast<uint32_t>(fmin(fmax(qv, 0.0), 15.0));
                }
                packed |= code << (4 * i);
            }
            *reinterpret_cast<uint16_t*>(codes + row * kRowBytes + lane * 2) =
                static_cast<uint16_t>(packed);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) count += __shfl_xor_sync(0xffffffffu, count, o);
    if (exceeded != nullptr && lane == 0) exceeded[pair] = count;
}


// ---------------------------------------------------------------------------
// Steps 1-2 in one launch: one thread-block cluster of C CTAs per
// (sequence, KV head) keeps the head's fp64 centroids in shared memory, so
// nothing goes through global memory but the keys read and the codes
// written.
//   build:    CTA r takes a contiguous 1/C of the head's blocks; each
//             half-warp takes one block at a time, lane l (of 16) owns
//             channels 8l .. 8l+7 and reads 16 bytes of every key row (a
//             half-warp reads a whole 256-byte row per instruction, the 16
//             rows of a page in flight at once).  Token-order fp64 sums, as
//             in the two-pass build.  Each CTA's per-channel min / max:
//             across the two half-warps of a warp by shuffle, across warps
//             by shared-memory atomics on order-mapped keys.
//   exchange: every CTA sends its 128 mins and 128 maxes to every CTA of
//             the cluster (16-byte asynchronous stores counted on the
//             receiver's mbarrier); all CTAs then hold the head's min / max
//             and derive the same scale / zero point.
//   quantize: every CTA codes its own rows from shared memory.
// A head fits when its centroid capacity is at most C x kFusedRows rows; a
// layer with a larger head takes the two-pass kernels.
constexpr int kFusedThreads = 512;
constexpr int kFusedHalfWarps = kFusedThreads / 16;
constexpr int kFusedRows = 160;                 // fp64 centroid rows per CTA


__device__ __forceinline__ void st_async_u4(uint32_t remote_addr, uint4 v, uint32_t remote_bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, "
        "[%5];" ::"r"(remote_addr),
        "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(remote_bar)
        : "memory");
}

__global__ void __launch_bounds__(kFusedThreads, 1)
    centroid_fused_kernel(const KvDesc kv, int32_t* err, int rows_cap, uint8_t* __restrict__ codes,
                          float* __restrict__ scale_out, int32_t* __restrict__ zp_out,
                          int format) {
    extern __shared__ __align__(16) uint8_t fsm[];
    const uint32_t C = cluster_nctarank(), rank = cluster_ctarank();
    const int pair = blockIdx.x / C;
    const int s = pair / kv.Hkv, h = pair % kv.Hkv;
    const int tid = threadIdx.x;
    const int hw = tid >> 4, hl = tid & 15;      // half-warp, lane within it
    const bool int4 = format != ABSP_CENTROIDS_BF16;
    double* cent = reinterpret_cast<double*>(fsm);                            // [rows_cap][128]
    double* recv = cent + static_cast<size_t>(rows_cap) * kD;                 // [C][2][128]
    unsigned long long* red = reinterpret_cast<unsigned long long*>(recv + C * 2 * kD);  // [2][128]
    double* par = reinterpret_cast<double*>(red + 2 * kD);                   // scale, zp [2][128]
    int32_t* pg = reinterpret_cast<int32_t*>(par + 2 * kD);                   // [rows_cap * 4]
    unsigned long long* bar = reinterpret_cast<unsigned long long*>(pg + rows_cap * 4);
    const uint32_t bar_a = smem_u32(bar);

    if (tid == 0) {
        mbar_init(bar_a, 1);
        fence_mbar_init();
        // every other CTA's 128 mins and 128 maxes
        if (int4 && C > 1) mbar_arrive_expect_tx(bar_a, (C - 1) * 2 * kD * 8);
    }
    if (tid < kD) {
        red[tid] = ~0ull;        // min keys
        red[kD + tid] = 0ull;    // max keys
    }
    // release: the barrier set-up is visible cluster-wide once the matching
    // wait (before the first remote store) completes
    cluster_arrive();

    int len = kv.seq_lens[s];
    if (len < 0 || len > kv.max_pages * kPage) {
        if (tid == 0 && rank == 0 && h == 0) set_error(err, ABSP_ERR_DEVICE_FAULT, s);
        len = 0;
    }
    const int bs = kv.bs[h];
    const int spb = bs / kPage;
    const int n = (len + bs - 1) / bs;
    const int per = (n + static_cast<int>(C) - 1) / static_cast<int>(C);  // <= rows_cap
    const int r0 = min(n, static_cast<int>(rank) * per);
    const int nrows = min(n, r0 + per) - r0;
    const int npg = (len + kPage - 1) / kPage;
    // page ids of this CTA's blocks, read once, in parallel
    const int32_t* pt = kv.page_table + static_cast<int64_t>(s) * kv.max_pages;
    for (int i = tid; i < nrows * spb; i += kFusedThreads) {
        const int lp = r0 * spb + i;
        pg[i] = lp < npg ? pt[lp] : -1;
    }
    __syncthreads();

    // ---- build: token-order fp64 sums, one block per half-warp at a time
    for (int r = hw; r < nrows; r += kFusedHalfWarps) {
        const int b = r0 + r;
        const int t0 = b * bs;
        const int cnt = min(bs, len - t0);
        double a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = 0.0;
        for (int j = 0; j * kPage < cnt; ++j) {
            const int nt = min(kPage, cnt - j * kPage);
            const int phys = pg[r * spb + j];
            if (phys < 0 || phys >= kv.num_phys_pages) {
                if (hl == 0) set_error(err, ABSP_ERR_DEVICE_FAULT, s);
                continue;
            }
            const __nv_bfloat16* src =
                kv.k_pages + ((static_cast<int64_t>(phys) * kv.Hkv + h) * kPage) * kD + hl * 8;
            uint4 v[kPage];
#pragma unroll
            for (int t = 0; t < kPage; ++t)
                if (t < nt) v[t] = ld_nc_u4(src + t * kD);
#pragma unroll
            for (int t = 0; t < kPage; ++t) {
                if (t < nt) {
                    a[0] += static_cast<double>(bf16lo(v[t].x));
                    a[1] += static_cast<double>(bf16hi(v[t].x));
                    a[2] += static_cast<double>(bf16lo(v[t].y));
                    a[3] += static_cast<double>(bf16hi(v[t].y));
                    a[4] += static_cast<double>(bf16lo(v[t].z));
                    a[5] += static_cast<double>(bf16hi(v[t].z));
                    a[6] += static_cast<double>(bf16lo(v[t].w));
                    a[7] += static_cast<double>(bf16hi(v[t].w));
                }
            }
        }
        // 2^-k for cnt = 2^k (used only then)
        const double dinv = __hiloint2double((1023 - (__ffs(cnt) - 1)) << 20, 0);
        double2* dst = reinterpret_cast<double2*>(cent + static_cast<size_t>(r) * kD + hl * 8);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            dst[i] = make_double2(mean_of(a[2 * i], cnt, dinv), mean_of(a[2 * i + 1], cnt, dinv));
    }
    __syncthreads();

    if (int4) {
        // ---- this CTA's per-channel min / max over its rows in shared
        // memory (thread t: channel t % 128, every 4th row), then the
        // cluster's
        {
            const int d = tid & (kD - 1), q4 = tid >> 7;
            double mn = __longlong_as_double(0x7FF0000000000000ll), mx = -mn;
            for (int r = q4; r < nrows; r += kFusedThreads / kD) {
                const double c = cent[static_cast<size_t>(r) * kD + d];
                mn = fmin(mn, c);
                mx = fmax(mx, c);
            }
            if (mn <= mx) {
                atomicMin(&red[d], ord_f64(mn));
                atomicMax(&red[kD + d], ord_f64(mx));
            }
        }
        __syncthreads();
        cluster_wait();   // every CTA's barrier is initialised
        // 256 doubles (mins, then maxes) = 128 pieces of 16 bytes to every
        // CTA; a CTA with no block sends the +inf / -inf sentinels
        for (int i = tid; i < static_cast<int>(C) * 128; i += kFusedThreads) {
            const uint32_t dst_rank = static_cast<uint32_t>(i / 128);
            const int piece = i % 128;
            const int k0 = 2 * piece;
            auto val = [&](int k) -> double {
                const unsigned long long key = red[k];
                if (k < kD ? key == ~0ull : key == 0ull)
                    return k < kD ? __longlong_as_double(0x7FF0000000000000ll)
                                  : __longlong_as_double(static_cast<long long>(0xFFF0000000000000ull));
                return unord_f64(key);
            };
            const double d0 = val(k0), d1 = val(k0 + 1);
            double* slot = recv + (rank * 2) * kD + k0;
            if (dst_rank == rank) {
                slot[0] = d0;
                slot[1] = d1;
            } else {
                uint4 u;
                u.x = static_cast<uint32_t>(__double_as_longlong(d0));
                u.y = static_cast<uint32_t>(static_cast<unsigned long long>(__double_as_longlong(d0)) >> 32);
                u.z = static_cast<uint32_t>(__double_as_longlong(d1));
                u.w = static_cast<uint32_t>(static_cast<unsigned long long>(__double_as_longlong(d1)) >> 32);
                st_async_u4(dsmem_addr(smem_u32(slot), dst_rank), u, dsmem_addr(bar_a, dst_rank));
            }
        }
        if (C > 1) {
            // bounded wait: every other CTA's (min, max) has arrived
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait_cluster(bar_a, 0)) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    set_error(err, ABSP_ERR_TIMEOUT, 6);
                    break;
                }
            }
        }
        __syncthreads();
        if (tid < kD) {
            const int d = tid;
            double lo = recv[d], hi = recv[kD + d];
            for (uint32_t r = 1; r < C; ++r) {
                lo = fmin(lo, recv[(2 * r) * kD + d]);
                hi = fmax(hi, recv[(2 * r + 1) * kD + d]);
            }
            double sc = 0.0, z = 0.0;
            float scf = 0.0f;
            int32_t zi = 0;
            if (n > 0 && hi > lo) {
                const float f = __double2float_rn((hi - lo) / 15.0);
                if (f > 0.0f) {
                    scf = f;
                    sc = static_cast<double>(f);
                    double zr = rint(-lo / sc);
                    zr = fmin(fmax(zr, -2147483648.0), 2147483647.0);
                    zi = static_cast<int32_t>(zr);
                    z = static_cast<double>(zi);
                }
            }
            par[d] = sc;
            par[kD + d] = z;
            if (rank == 0) {
                const int64_t pi = (static_cast<int64_t>(s) * kv.Hkv + h) * kD + d;
                scale_out[pi] = scf;
                zp_out[pi] = zi;
            }
        }
    } else {
        cluster_wait();
    }
    __syncthreads();

    // ---- store: INT4 codes (4 bytes per lane) or bf16 rows (16 bytes)
    const int64_t row0 = static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h] + r0;
    double sc[8], zz[8], iv[8];
    if (int4) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            sc[i] = par[hl * 8 + i];
            zz[i] = par[kD + hl * 8 + i];
            iv[i] = sc[i] != 0.0 ? 1.0 / sc[i] : 0.0;
        }
    }
    for (int r = hw; r < nrows; r += kFusedHalfWarps) {
        const double2* src = reinterpret_cast<const double2*>(cent + static_cast<size_t>(r) * kD + hl * 8);
        double c[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double2 u = src[i];
            c[2 * i] = u.x;
            c[2 * i + 1] = u.y;
        }
        if (int4) {
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t code = 0;
                if (sc[i] != 0.0) {
                    double qv = rint_div(c[i], sc[i], iv[i]) + zz[i];
                    qv = fmin(fmax(qv, 0.0), 15.0);
                    code = static_cast<uint32_t>(qv);
                }
                packed |= code << (4 * i);
            }
            *reinterpret_cast<uint32_t*>(codes + (row0 + r) * kRowBytes + hl * 4) = packed;
        } else {
            uint4 o;
            o.x = f64_to_bf16_rne(c[0]) | (f64_to_bf16_rne(c[1]) << 16);
            o.y = f64_to_bf16_rne(c[2]) | (f64_to_bf16_rne(c[3]) << 16);
            o.z = f64_to_bf16_rne(c[4]) | (f64_to_bf16_rne(c[5]) << 16);
            o.w = f64_to_bf16_rne(c[6]) | (f64_to_bf16_rne(c[7]) << 16);
            *reinterpret_cast<uint4*>(codes + (row0 + r) * (2 * kD) + hl * 16) = o;
        }
    }
}

}  // namespace

size_t build_ws_bytes(const KvDesc& kv) {
    const size_t mm = static_cast<size_t>(kv.S) * kv.Hkv * kD * 2 * sizeof(unsigned long long);
    const size_t cent = static_cast<size_t>(kv.S) * kv.rows_per_seq * kD * sizeof(double);
    return kWsHeader + mm + cent;
}

BuildWs build_ws_layout(void* ws, const KvDesc& kv) {
    uint8_t* p = static_cast<uint8_t*>(ws);
    BuildWs w;
    w.err = reinterpret_cast<int32_t*>(p);
    w.minmax = reinterpret_cast<unsigned long long*>(p + kWsHeader);
    const size_t mm = static_cast<size_t>(kv.S) * kv.Hkv * kD * 2 * sizeof(unsigned long long);
    w.cent = reinterpret_cast<double*>(p + kWsHeader + mm);
    return w;
}

static dim3 chunk_grid(const KvDesc& kv) {
    const int chunks = (kv.max_pages * kPage + kChunkTokens - 1) / kChunkTokens;
    return dim3(chunks, kv.Hkv, kv.S);
}

cudaError_t launch_build(const KvDesc& kv, const BuildWs& w, cudaStream_t st) {
    // order-mapped sentinels: every key (min of c, and min of -c for the
    // max) starts at all-ones
    const size_t pairs = static_cast<size_t>(kv.S) * kv.Hkv * kD;
    cudaError_t e = cudaMemsetAsync(w.minmax, 0xFF, 2 * pairs * sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static bool configured[16] = {};
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        // one-time attribute set-up; relaxed capture mode lets it through
        // while the caller captures `st` (it touches no stream)
        cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
        cudaThreadExchangeStreamCaptureMode(&mode);
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 16 || !configured[dev]) {
            e = cudaFuncSetAttribute(centroid_build_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kBuildSmem);
            if (e == cudaSuccess && dev >= 0 && dev < 16) configured[dev] = true;
        }
        cudaThreadExchangeStreamCaptureMode(&mode);
        if (e != cudaSuccess) return e;
    }
    centroid_build_kernel<<<chunk_grid(kv), kBuildWarps * 32, kBuildSmem, st>>>(kv, w);
    return cudaGetLastError();
}

cudaError_t launch_append(const KvDesc& kv, uint8_t* codes, const float* scale, const int32_t* zp,
                          int format, int32_t* exceeded, int32_t* err, cudaStream_t st) {
    const int pairs = kv.S * kv.Hkv;
    centroid_append_kernel<<<(pairs + kBuildWarps - 1) / kBuildWarps, kBuildWarps * 32, 0, st>>>(
        kv, codes, scale, zp, format, exceeded, err);
    return cudaGetLastError();
}

cudaError_t launch_quantize(const KvDesc& kv, const BuildWs& w, uint8_t* codes, float* scale,
                            int32_t* zp, int format, cudaStream_t st) {
    if (format == ABSP_CENTROIDS_BF16)
        centroid_bf16_kernel<<<chunk_grid(kv), kBuildWarps * 32, 0, st>>>(kv, w, codes);
    else
        centroid_quantize_kernel<<<chunk_grid(kv), kBuildWarps * 32, 0, st>>>(kv, w, codes, scale,
                                                                           zp);
    return cudaGetLastError();
}


size_t fused_smem_bytes(int rows_cap, int C) {
    return static_cast<size_t>(rows_cap) * kD * 8 + static_cast<size_t>(C) * 2 * kD * 8 +
           2 * kD * 8 + 2 * kD * 8 + static_cast<size_t>(rows_cap) * 4 * 4 + 16;
}

// Cluster size of the fused build, or 0 when some head's centroids do not
// fit on one cluster (the two-pass kernels then run instead).
int fused_cluster(const KvDesc& kv, int num_sms, int* rows_cap) {
    int cap = 0;
    for (int h = 0; h < kv.Hkv; ++h) cap = std::max(cap, kv.cap[h]);
    int C = 1;
    while (C < 16 && (cap + C - 1) / C > kFusedRows) C *= 2;
    if ((cap + C - 1) / C > kFusedRows) return 0;
    const int pairs = kv.S * kv.Hkv;
    // more CTAs per head while the launch still fits in one wave
    while (C < 16 && pairs * C * 2 <= num_sms) C *= 2;
    *rows_cap = (cap + C - 1) / C;
    return C;
}

cudaError_t launch_build_quantize(const KvDesc& kv, const BuildWs& w, uint8_t* codes, float* scale,
                                  int32_t* zp, int format, cudaStream_t st) {
    static std::mutex mu;
    static bool configured[16] = {};
    int dev = 0, num_sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        num_sms = 148;
    int rows_cap = 0;
    int C = fused_cluster(kv, num_sms, &rows_cap);
    if (C > 0) {
        cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
        cudaThreadExchangeStreamCaptureMode(&mode);
        {
            std::lock_guard<std::mutex> lock(mu);
            if (dev < 0 || dev >= 16 || !configured[dev]) {
                e = cudaFuncSetAttribute(centroid_fused_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(centroid_fused_kernel,
                                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
                if (e == cudaSuccess && dev >= 0 && dev < 16) configured[dev] = true;
            }
        }
        cudaThreadExchangeStreamCaptureMode(&mode);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kv.S * kv.Hkv * C);
        cfg.blockDim = dim3(kFusedThreads);
        cfg.dynamicSmemBytes = fused_smem_bytes(rows_cap, C);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, centroid_fused_kernel, kv, w.err, rows_cap, codes, scale,
                                  zp, format);
    }
    e = launch_build(kv, w, st);
    if (e != cudaSuccess) return e;
    return launch_quantize(kv, w, codes, scale, zp, format, st);
}

}  // namespace absp
