// Steps 1-2 of AB-Sparse (arXiv 2605.12110): mean-key block centroids
// (Fig. 1 "block representation"; Fig. 5: centroids are built over all key
// vectors of a head, once) and their INT4 asymmetric per-channel codes
// (Fig. 8).
//
// Kernel shapes.  The build tiles a layer by (1024-token chunk, KV head,
// sequence): every CTA covers the same number of tokens whatever the head's
// block size (64, 32 or 16 blocks), so work is balanced across heads.
//   build:    one half-warp per block; lane l owns channels 8l..8l+7 and
//             reads 16 bytes of every key row (a half-warp reads a whole
//             256-byte row per instruction).  The sums equal the token-order
//             fp64 sums bit for bit (block_sums).  The CTA reduces its
//             per-channel min / max in shared memory and issues one atomic
//             per channel (order-mapped fp64 keys).
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

// The INT4 code clamp(rint(c / sc) + zp, 0, 15) (IEEE division, round half
// to even, fp64) without dividing on the common path: r = c * inv (inv =
// 1 / sc rounded) and the rounded quotient are both within about 2^-52 |r|
// of c / sc, under 2^-31 for |r| < 2^20, so when r lies at least 2^-28 from
// every half-integer (|r - rint(r)| <= 0.5 - 2^-28) both round to the same
// integer; the offset and clamp then run on integers.  Larger quotients and
// residues nearer 0.5 take the exact path.
__device__ __forceinline__ uint32_t int4_code(double c, double sc, double inv, int32_t zp) {
    const double r = c * inv;
    const double fl = rint(r);
    if (fabs(r) < 0x1p20 && fabs(r - fl) <= 0.5 - 0x1p-28) {
        const long long v = static_cast<long long>(fl) + zp;
        return static_cast<uint32_t>(v < 0 ? 0 : v > 15 ? 15 : v);
    }
    const double qv = fmin(fmax(rint(c / sc) + static_cast<double>(zp), 0.0), 15.0);
    return static_cast<uint32_t>(qv);
}

// INT4 parameters of one channel from its order-mapped min key and the key
// of its negated max (Fig. 8): scf = fp32((max - min) / 15) and, in fp64,
// sc = scf and zi = rint(-min / sc) saturated to int32; a channel with
// max == min, or a (sequence, head) with no rows (any = false), gets 0 / 0.
__device__ __forceinline__ void channel_params(unsigned long long kmn, unsigned long long knmx,
                                               bool any, float& scf, double& sc, int32_t& zi) {
    scf = 0.0f;
    sc = 0.0;
    zi = 0;
    if (!any) return;
    const double mn = unord_f64(kmn);
    const double mx = -unord_f64(knmx);
    if (mx > mn) {
        const float f = __double2float_rn((mx - mn) / 15.0);
        if (f > 0.0f) {
            scf = f;
            sc = static_cast<double>(f);
            double zr = rint(-mn / sc);
            zr = fmin(fmax(zr, -2147483648.0), 2147483647.0);
            zi = static_cast<int32_t>(zr);
        }
    }
}

// ---------------------------------------------------------------------------
// Exact block sums of bf16 keys.
//
// The centroid of a block is the token-order fp64 sum of its keys over the
// token count.  That sum is exact, and so equal to the sum in any order,
// whenever the block's nonzero values span few enough binades: a bf16 value
// with biased exponent e is a multiple of 2^(e-134) below 2^(e-126), so with
// exponents in [emin, emax] and at most 64 tokens every partial sum is a
// multiple of 2^(emin-134) below 2^(emax-120), and fp64 holds it exactly
// when emax - emin <= 39.  Under that condition a page's 16 rows may be
// summed in any exact way.  The fast path sums them in fp32 twice, rounded
// down and rounded up: each rounded sum bounds the exact one from its side
// (also through further additions of such bounds, each rounded the same
// way), so where the two agree both are exact.  One fp32 -> fp64 conversion
// per page and channel then replaces sixteen.  A page whose two sums differ
// is summed in fp64 instead; a block that fails the exponent condition (or
// holds a zero, subnormal, infinite or NaN key) is summed again in token
// order, as the definition reads.

// One word of a key row (two bf16 keys, channels c and c+1) into the
// fast path's state: both keys widened to fp32 and added to the round-down
// and round-up sums (packed pairs, low channel first), and the keys'
// magnitudes (bf16 bits without the sign, as 16-bit integers: ordered as
// the values' magnitudes, NaN above infinity) folded into the running
// min / max.  One asm block, so that each word is consumed as it arrives.
__device__ __forceinline__ void fold_word(uint64_t& dn, uint64_t& up, uint32_t& mn, uint32_t& mx,
                                          uint32_t w) {
    asm("{\n\t"
        ".reg .b32 lo, hi, m;\n\t"
        ".reg .b64 f;\n\t"
        "shl.b32 lo, %4, 16;\n\t"
        "and.b32 hi, %4, 0xFFFF0000;\n\t"
        "mov.b64 f, {lo, hi};\n\t"
        "add.rm.f32x2 %0, %0, f;\n\t"
        "add.rp.f32x2 %1, %1, f;\n\t"
        "and.b32 m, %4, 0x7FFF7FFF;\n\t"
        "min.u16x2 %2, %2, m;\n\t"
        "max.u16x2 %3, %3, m;\n\t"
        "}"
        : "+l"(dn), "+l"(up), "+r"(mn), "+r"(mx)
        : "r"(w));
}

__device__ __forceinline__ float f32x2_lo(uint64_t v) {
    return __uint_as_float(static_cast<uint32_t>(v));
}

__device__ __forceinline__ float f32x2_hi(uint64_t v) {
    return __uint_as_float(static_cast<uint32_t>(v >> 32));
}

// Channels 8hl .. 8hl+7 of a block's cnt keys summed into a[] (pages[j]
// is the block's j-th page), bit-identical to the token-order fp64 sums.
// The first pass takes the fast path page by page; a page whose two fp32
// sums differ is read again and added to a[] in fp64 token by token (exact
// under the exponent condition, checked at the end).  If the condition
// fails, a second pass sums the block in token order throughout.  Both
// passes share one load site, so the rare branches hold no registers of
// their own.
__device__ __forceinline__ void block_sums(const KvDesc& kv, const int32_t* pages, int h, int hl,
                                           int cnt, int s, int32_t* err, double a[8]) {
    bool ordered = false;   // second pass: the definition, term by term
    for (;;) {
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = 0.0;
        uint32_t mn = 0xFFFFFFFFu, mx = 0u;   // |key| extremes over the block, 16-bit pairs
        for (int j = 0; j * kPage < cnt; ++j) {
            const int nt = min(kPage, cnt - j * kPage);
            const int phys = pages[j];
            if (phys < 0 || phys >= kv.num_phys_pages) {
                if (hl == 0) set_error(err, ABSP_ERR_DEVICE_FAULT, s);
                continue;
            }
            const __nv_bfloat16* src =
                kv.k_pages + ((static_cast<int64_t>(phys) * kv.Hkv + h) * kPage) * kD + hl * 8;
            bool slow = ordered;
            for (;;) {
                uint4 v[kPage];
#pragma unroll
                for (int t = 0; t < kPage; ++t)
                    if (t < nt) v[t] = ld_nc_u4(src + t * kD);
                if (slow) {
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
                    break;
                }
                uint64_t dn[4] = {0, 0, 0, 0}, up[4] = {0, 0, 0, 0};
#pragma unroll
                for (int t = 0; t < kPage; ++t) {
                    if (t < nt) {
                        fold_word(dn[0], up[0], mn, mx, v[t].x);
                        fold_word(dn[1], up[1], mn, mx, v[t].y);
                        fold_word(dn[2], up[2], mn, mx, v[t].z);
                        fold_word(dn[3], up[3], mn, mx, v[t].w);
                    }
                }
                bool exact = true;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    exact = exact && f32x2_lo(dn[i]) == f32x2_lo(up[i]) &&
                            f32x2_hi(dn[i]) == f32x2_hi(up[i]);
                if (exact) {
                    // the round-up sums: +0 where an exact sum is zero, as in fp64
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        a[2 * i] += static_cast<double>(f32x2_lo(up[i]));
                        a[2 * i + 1] += static_cast<double>(f32x2_hi(up[i]));
                    }
                    break;
                }
                slow = true;
            }
        }
        if (ordered) return;
        const int emin = static_cast<int>(min(mn & 0xFFFFu, mn >> 16) >> 7);
        const int emax = static_cast<int>(max(mx & 0xFFFFu, mx >> 16) >> 7);
        bool ok = emin >= 1 && emax <= 254 && emax - emin <= 39;
#pragma unroll
        for (int i = 0; i < 8; ++i) ok = ok && a[i] == a[i];
        if (ok) return;
        ordered = true;
    }
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

// One 1024-token chunk of (sequence s, KV head h), by one CTA of
// kBuildWarps warps.  Each half-warp takes one block at a time; lane l (of
// 16) owns channels 8l .. 8l+7 and reads 16 bytes of every key row (a
// half-warp reads a whole 256-byte row per instruction, a page's 16 rows in
// flight).  Sums as block_sums.  With bf16_rows the centroids are stored
// there rounded to bf16 and nothing else is done; otherwise they go to the
// workspace and to shared memory, and the chunk's per-channel min / max,
// taken over the shared copy, is merged with one atomic per channel into
// order-mapped keys (the max as the key of its negation, so that one fill
// of ones initialises every key).
__global__ void __launch_bounds__(kBuildWarps * 32)
    centroid_build_kernel(const KvDesc kv, BuildWs w, uint8_t* __restrict__ bf16_rows) {
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
    const int64_t row0 = static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h];

    for (int b = b_begin + hw; b < b_end; b += kHalfWarps) {
        const int t0 = b * bs;
        const int cnt = min(bs, len - t0);
        double a[8];
        block_sums(kv, pt + t0 / kPage, h, hl, cnt, s, w.err, a);
        // 2^-k for cnt = 2^k (used only then)
        const double dinv = __hiloint2double((1023 - (__ffs(cnt) - 1)) << 20, 0);
        double c[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = mean_of(a[i], cnt, dinv);
        if (bf16_rows != nullptr) {
            uint4 o;
            o.x = f64_to_bf16_rne(c[0]) | (f64_to_bf16_rne(c[1]) << 16);
            o.y = f64_to_bf16_rne(c[2]) | (f64_to_bf16_rne(c[3]) << 16);
            o.z = f64_to_bf16_rne(c[4]) | (f64_to_bf16_rne(c[5]) << 16);
            o.w = f64_to_bf16_rne(c[6]) | (f64_to_bf16_rne(c[7]) << 16);
            *reinterpret_cast<uint4*>(bf16_rows + (row0 + b) * (2 * kD) + hl * 16) = o;
            continue;
        }
        double2* dg = reinterpret_cast<double2*>(w.cent + (row0 + b) * kD + hl * 8);
        double2* ds = reinterpret_cast<double2*>(&rows_s[b - b_begin][hl * 8]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double2 v = make_double2(c[2 * i], c[2 * i + 1]);
            dg[i] = v;
            ds[i] = v;
        }
    }
    if (bf16_rows != nullptr) return;  // uniform
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

// Quantise: one CTA per (group of `rows_per_cta` rows, a multiple of 32 up
// to kQuantRows, KV head, sequence), launched as a programmatic dependent
// of the build so that it is resident when the build ends; it waits for
// the build's results before reading them.  Threads 0..127 derive the
// per-channel parameters (fp64 divisions) while the first rows' loads are
// in flight.  Warp w codes rows w, w + 8, ...
// of the group four at a time, the next four's loads issued before the
// current four are coded; lane L takes channels 4L .. 4L+3 and writes 2
// bytes of each 64-byte row.
constexpr int kQuantRows = 256;

__global__ void __launch_bounds__(kBuildWarps * 32)
    centroid_quantize_kernel(const KvDesc kv, BuildWs w, uint8_t* __restrict__ codes,
                             float* __restrict__ scale_out, int32_t* __restrict__ zp_out,
                             int rows_per_cta) {
    const int grp = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ double s_par[3][kD];   // scale, zero point, 1 / scale

    const int len = checked_len(kv, s, w.err);
    const int bs = kv.bs[h];
    const int n = len > 0 ? (len + bs - 1) / bs : 0;
    const int r_begin = grp * rows_per_cta;
    if (grp > 0 && r_begin >= n) return;  // uniform over the CTA
    const int r_end = min(n, r_begin + rows_per_cta);
    pdl_wait();                           // the build's rows and keys
    const int64_t row0 = static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h];

    constexpr int kRows = 4;
    constexpr int kStep = kRows * kBuildWarps;
    double c0[kRows][4], c1[kRows][4];
    auto load = [&](int b0, double (&cb)[kRows][4]) {
#pragma unroll
        for (int q = 0; q < kRows; ++q) {
            const int b = b0 + q * kBuildWarps;
            if (b < r_end) {
                const double2* src =
                    reinterpret_cast<const double2*>(w.cent + (row0 + b) * kD + lane * 4);
                const double2 u = src[0], v = src[1];
                cb[q][0] = u.x;
                cb[q][1] = u.y;
                cb[q][2] = v.x;
                cb[q][3] = v.y;
            }
        }
    };
    load(r_begin + warp, c0);

    if (threadIdx.x < kD) {
        const int d = threadIdx.x;
        const int64_t pi = (static_cast<int64_t>(s) * kv.Hkv + h) * kD + d;
        const int64_t pairs = static_cast<int64_t>(kv.S) * kv.Hkv * kD;
        float scf;
        double sc;
        int32_t zi;
        channel_params(n > 0 ? w.minmax[pi] : 0ull, n > 0 ? w.minmax[pairs + pi] : 0ull, n > 0,
                       scf, sc, zi);
        s_par[0][d] = sc;
        s_par[1][d] = static_cast<double>(zi);
        s_par[2][d] = sc != 0.0 ? 1.0 / sc : 0.0;
        if (grp == 0) {
            scale_out[pi] = scf;
            zp_out[pi] = zi;
        }
    }
    __syncthreads();
    double sc[4], iv[4];
    int32_t zi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sc[i] = s_par[0][lane * 4 + i];
        zi[i] = static_cast<int32_t>(s_par[1][lane * 4 + i]);   // an int32 held exactly
        iv[i] = s_par[2][lane * 4 + i];
    }
    auto code_rows = [&](int b0, const double (&cb)[kRows][4]) {
#pragma unroll
        for (int q = 0; q < kRows; ++q) {
            const int b = b0 + q * kBuildWarps;
            if (b >= r_end) break;
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t code = sc[i] != 0.0 ? int4_code(cb[q][i], sc[i], iv[i], zi[i]) : 0u;
                packed |= code << (4 * i);
            }
            *reinterpret_cast<uint16_t*>(codes + (row0 + b) * kRowBytes + lane * 2) =
                static_cast<uint16_t>(packed);
        }
    };
    // two buffers, named, so that every index is static
    for (int b0 = r_begin + warp; b0 < r_end; b0 += 2 * kStep) {
        if (b0 + kStep < r_end) load(b0 + kStep, c1);
        code_rows(b0, c0);
        if (b0 + kStep >= r_end) break;
        if (b0 + 2 * kStep < r_end) load(b0 + 2 * kStep, c0);
        code_rows(b0 + kStep, c1);
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


}  // namespace

// [header][min / max keys][fp64 rows]
static size_t minmax_bytes(const KvDesc& kv) {
    return static_cast<size_t>(kv.S) * kv.Hkv * kD * 2 * sizeof(unsigned long long);
}

size_t build_ws_bytes(const KvDesc& kv) {
    const size_t cent = static_cast<size_t>(kv.S) * kv.rows_per_seq * kD * sizeof(double);
    return kWsHeader + minmax_bytes(kv) + cent;
}

BuildWs build_ws_layout(void* ws, const KvDesc& kv) {
    uint8_t* p = static_cast<uint8_t*>(ws);
    BuildWs w;
    w.err = reinterpret_cast<int32_t*>(p);
    w.minmax = reinterpret_cast<unsigned long long*>(p + kWsHeader);
    w.cent = reinterpret_cast<double*>(p + kWsHeader + minmax_bytes(kv));
    return w;
}

static dim3 chunk_grid(const KvDesc& kv) {
    const int chunks = (kv.max_pages * kPage + kChunkTokens - 1) / kChunkTokens;
    return dim3(chunks, kv.Hkv, kv.S);
}

// The build kernel, writing fp64 rows + min / max keys (after one fill of
// ones over the keys), or, with bf16_rows, bf16 rows only.
static cudaError_t launch_build_rows(const KvDesc& kv, const BuildWs& w, uint8_t* bf16_rows,
                                     cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    if (bf16_rows == nullptr &&
        (e = cudaMemsetAsync(w.minmax, 0xFF, minmax_bytes(kv), st)) != cudaSuccess)
        return e;
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
    centroid_build_kernel<<<chunk_grid(kv), kBuildWarps * 32, bf16_rows ? 0 : kBuildSmem, st>>>(
        kv, w, bf16_rows);
    return cudaGetLastError();
}

cudaError_t launch_build(const KvDesc& kv, const BuildWs& w, cudaStream_t st) {
    return launch_build_rows(kv, w, nullptr, st);
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
    if (format == ABSP_CENTROIDS_BF16) {
        centroid_bf16_kernel<<<chunk_grid(kv), kBuildWarps * 32, 0, st>>>(kv, w, codes);
    } else {
        // rows per CTA: enough CTAs to fill the GPU a few times over, each
        // with whole 32-row steps
        int cap = 1, dev = 0, num_sms = 148;
        for (int h = 0; h < kv.Hkv; ++h) cap = std::max(cap, kv.cap[h]);
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            num_sms = 148;
        const long long rows = static_cast<long long>(kv.S) * kv.rows_per_seq;
        const long long want = (rows / (4ll * num_sms) + 31) / 32 * 32;
        const int rpc = static_cast<int>(std::min<long long>(kQuantRows, std::max(32ll, want)));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((cap + rpc - 1) / rpc, kv.Hkv, kv.S);
        cfg.blockDim = dim3(kBuildWarps * 32);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, centroid_quantize_kernel, kv, w, codes, scale, zp, rpc);
    }
    return cudaGetLastError();
}


cudaError_t launch_build_quantize(const KvDesc& kv, const BuildWs& w, uint8_t* codes, float* scale,
                                  int32_t* zp, int format, cudaStream_t st) {
    // BF16: the build writes the rows itself, one launch
    if (format == ABSP_CENTROIDS_BF16) return launch_build_rows(kv, w, codes, st);
    cudaError_t e = launch_build(kv, w, st);
    if (e != cudaSuccess) return e;
    return launch_quantize(kv, w, codes, scale, zp, format, st);
}

}  // namespace absp
