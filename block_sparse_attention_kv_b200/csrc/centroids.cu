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
#include "absp_internal.cuh"

namespace absp {

namespace {

constexpr int kChunkTokens = 1024;
constexpr int kBuildWarps = 8;

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

__global__ void __launch_bounds__(kBuildWarps * 32)
    centroid_build_kernel(const KvDesc kv, BuildWs w) {
    const int chunk = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ double red_min[kBuildWarps][kD];
    __shared__ double red_max[kBuildWarps][kD];

    const int len = checked_len(kv, s, w.err);
    const int tok0 = chunk * kChunkTokens;
    if (len <= tok0) return;  // uniform over the CTA

    const int bs = kv.bs[h];
    const int n = (len + bs - 1) / bs;
    const int b_begin = tok0 / bs;
    const int b_end = min(n, (tok0 + kChunkTokens) / bs);
    const int32_t* pt = kv.page_table + static_cast<int64_t>(s) * kv.max_pages;
    double* cent = w.cent + (static_cast<int64_t>(s) * kv.rows_per_seq + kv.row_base[h]) * kD;

    double mn[4], mx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        mn[i] = __longlong_as_double(0x7FF0000000000000ll);   // +inf
        mx[i] = -mn[i];
    }

    for (int b = b_begin + warp; b < b_end; b += kBuildWarps) {
        const int t0 = b * bs;
        const int cnt = min(bs, len - t0);
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        for (int tp = t0; tp < t0 + cnt; tp += kPage) {
            const int nt = min(kPage, t0 + cnt - tp);
            const int phys = pt[tp / kPage];
            if (phys < 0 || phys >= kv.num_phys_pages) {
                if (lane == 0) set_error(w.err, ABSP_ERR_DEVICE_FAULT, s);
                continue;
            }
            const __nv_bfloat16* src =
                kv.k_pages + ((static_cast<int64_t>(phys) * kv.Hkv + h) * kPage) * kD + lane * 4;
            uint2 v[kPage];
#pragma unroll
            for (int t = 0; t < kPage; ++t)
                if (t < nt) v[t] = ld_nc_u2(src + t * kD);
#pragma unroll
            for (int t = 0; t < kPage; ++t) {
                if (t < nt) {
                    a0 += static_cast<double>(bf16lo(v[t].x));
                    a1 += static_cast<double>(bf16hi(v[t].x));
                    a2 += static_cast<double>(bf16lo(v[t].y));
                    a3 += static_cast<double>(bf16hi(v[t].y));
                }
            }
        }
        const double dc = static_cast<double>(cnt);
        const double c0 = a0 / dc, c1 = a1 / dc, c2 = a2 / dc, c3 = a3 / dc;
        double2* dst = reinterpret_cast<double2*>(cent + static_cast<int64_t>(b) * kD + lane * 4);
        dst[0] = make_double2(c0, c1);
        dst[1] = make_double2(c2, c3);
        mn[0] = fmin(mn[0], c0); mx[0] = fmax(mx[0], c0);
        mn[1] = fmin(mn[1], c1); mx[1] = fmax(mx[1], c1);
        mn[2] = fmin(mn[2], c2); mx[2] = fmax(mx[2], c2);
        mn[3] = fmin(mn[3], c3); mx[3] = fmax(mx[3], c3);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        red_min[warp][lane * 4 + i] = mn[i];
        red_max[warp][lane * 4 + i] = mx[i];
    }
    __syncthreads();
    if (threadIdx.x < kD) {
        const int d = threadIdx.x;
        double lo = red_min[0][d], hi = red_max[0][d];
#pragma unroll
        for (int k = 1; k < kBuildWarps; ++k) {
            lo = fmin(lo, red_min[k][d]);
            hi = fmax(hi, red_max[k][d]);
        }
        if (lo <= hi) {
            const int64_t pi = (static_cast<int64_t>(s) * kv.Hkv + h) * kD + d;
            const int64_t pairs = static_cast<int64_t>(kv.S) * kv.Hkv * kD;
            atomicMin(w.minmax + pi, ord_f64(lo));
            atomicMax(w.minmax + pairs + pi, ord_f64(hi));
        }
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
            const double mx = unord_f64(w.minmax[pairs + pi]);
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
    double sc[4], zz[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sc[i] = s_scale[lane * 4 + i];
        zz[i] = s_zp[lane * 4 + i];
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
                double qv = rint(c[i] / sc[i]) + zz[i];
                qv = fmin(fmax(qv, 0.0), 15.0);
                code = static_cast<uint32_t>(qv);
            }
            packed |= code << (4 * i);
        }
        *reinterpret_cast<uint16_t*>(codes + (row0 + b) * kRowBytes + lane * 2) =
            static_cast<uint16_t>(packed);
    }
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
    // order-mapped sentinels: every min key starts at all-ones, every max
    // key at zero
    const size_t pairs = static_cast<size_t>(kv.S) * kv.Hkv * kD;
    cudaError_t e = cudaMemsetAsync(w.minmax, 0xFF, pairs * sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(w.minmax + pairs, 0, pairs * sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
    centroid_build_kernel<<<chunk_grid(kv), kBuildWarps * 32, 0, st>>>(kv, w);
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

}  // namespace absp
