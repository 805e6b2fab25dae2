// extern "C" entry points of libabsp: host-side validation, workspace
// layout, tensor-map encoding and the launches.  See include/absp.h for the
// contract of every call.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "absp_internal.cuh"
#include "absp_trace.h"

using namespace absp;

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

// Validate a layer description and fill the by-value kernel descriptor.
absp_status absp::make_desc(const absp_layer_kv* kv, KvDesc* d, bool need_v) {
    if (kv == nullptr || d == nullptr) return ABSP_ERR_INVALID_ARG;
    if (kv->head_dim != ABSP_HEAD_DIM || kv->page_size != ABSP_PAGE_SIZE)
        return ABSP_ERR_UNSUPPORTED;
    if (kv->num_seqs < 1 || kv->num_kv_heads < 1 || kv->num_q_heads < 1 ||
        kv->max_pages_per_seq < 1 || kv->num_phys_pages < 1)
        return ABSP_ERR_INVALID_ARG;
    if (kv->num_kv_heads > ABSP_MAX_KV_HEADS) return ABSP_ERR_UNSUPPORTED;
    if (kv->num_q_heads % kv->num_kv_heads != 0) return ABSP_ERR_INVALID_ARG;
    if (kv->num_q_heads / kv->num_kv_heads > ABSP_MAX_GROUP) return ABSP_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(kv->max_pages_per_seq) * ABSP_PAGE_SIZE > (1ll << 30))
        return ABSP_ERR_UNSUPPORTED;
    // tensor-map row coordinates are int32 (the first test keeps the
    // product below from overflowing)
    if (kv->num_phys_pages >= (1ll << 31) ||
        kv->num_phys_pages * kv->num_kv_heads * ABSP_PAGE_SIZE >= (1ll << 31))
        return ABSP_ERR_UNSUPPORTED;
    if (kv->seq_lens == nullptr || kv->page_table == nullptr || kv->k_pages == nullptr ||
        kv->block_size == nullptr || (need_v && kv->v_pages == nullptr))
        return ABSP_ERR_INVALID_ARG;
    if (!aligned(kv->k_pages, kAlign) || (need_v && !aligned(kv->v_pages, kAlign)))
        return ABSP_ERR_INVALID_ARG;
    std::memset(d, 0, sizeof(*d));
    d->S = kv->num_seqs;
    d->Hq = kv->num_q_heads;
    d->Hkv = kv->num_kv_heads;
    d->G = kv->num_q_heads / kv->num_kv_heads;
    d->max_pages = kv->max_pages_per_seq;
    d->num_phys_pages = kv->num_phys_pages;
    d->seq_lens = kv->seq_lens;
    d->page_table = kv->page_table;
    d->k_pages = static_cast<const __nv_bfloat16*>(kv->k_pages);
    d->v_pages = static_cast<const __nv_bfloat16*>(kv->v_pages);
    int64_t rows = 0;
    const int64_t tokens = static_cast<int64_t>(kv->max_pages_per_seq) * ABSP_PAGE_SIZE;
    for (int h = 0; h < kv->num_kv_heads; ++h) {
        const int bs = kv->block_size[h];
        if (bs != 16 && bs != 32 && bs != 64) return ABSP_ERR_INVALID_ARG;
        d->bs[h] = bs;
        d->cap[h] = static_cast<int32_t>((tokens + bs - 1) / bs);
        d->row_base[h] = static_cast<int32_t>(rows);
        rows += d->cap[h];
    }
    if (rows >= (1ll << 31)) return ABSP_ERR_UNSUPPORTED;
    d->rows_per_seq = rows;
    return ABSP_OK;
}

namespace {
thread_local int t_last_cuda = 0;  // last CUDA error turned into ABSP_ERR_CUDA here
}  // namespace

absp_status absp::cuda_status(int e) {
    if (e == 0) return ABSP_OK;
    t_last_cuda = e;
    return ABSP_ERR_CUDA;
}

namespace {

absp_status check_budget(const KvDesc& d, int32_t budget, int32_t* kmax, int32_t* nmax) {
    if (budget < ABSP_PAGE_SIZE || budget > ABSP_MAX_BUDGET) return ABSP_ERR_INVALID_ARG;
    int32_t km = 1, nm = 0;
    for (int h = 0; h < d.Hkv; ++h) {
        km = std::max(km, std::max(1, budget / d.bs[h]));
        nm = std::max(nm, d.cap[h]);
    }
    if (kmax) *kmax = km;
    if (nmax) *nmax = nm;
    return ABSP_OK;
}

absp_status from_cuda(cudaError_t e) { return cuda_status(static_cast<int>(e)); }

// ----------------------------------------------------------- tensor maps --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A [num_phys_pages * Hkv * 16][128] bf16 view of one page pool; a box is
// 16 token rows x 64 channels (128 bytes, 128-byte swizzle), so one
// (page, head) slice is two boxes.
absp_status page_tensor_map(const void* pages, const KvDesc& d, CUtensorMap* m) {
    // the encoding is a driver call: on a thread that has not used CUDA yet
    // no context is current, so let the runtime bind the current device's
    // context first (once per thread)
    static thread_local bool bound = false;
    if (!bound) {
        const cudaError_t e = cudaFree(nullptr);
        if (e != cudaSuccess) return from_cuda(e);
        bound = true;
    }
    auto fn = encode_fn();
    if (fn == nullptr) return cuda_status(cudaErrorNotSupported);
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(ABSP_HEAD_DIM),
                          static_cast<cuuint64_t>(d.num_phys_pages) * d.Hkv * ABSP_PAGE_SIZE};
    cuuint64_t strides[1] = {ABSP_HEAD_DIM * 2};
    cuuint32_t box[2] = {64, ABSP_PAGE_SIZE};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pages), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return cuda_status(static_cast<int>(r));  // a driver code (same numbering for the usual ones)
}

size_t decode_ws_bytes(const KvDesc& d) {
    const size_t act = round_up(static_cast<size_t>(d.S) * d.Hq * ABSP_HEAD_DIM * 2, kAlign);
    return kWsHeader + 2 * act;
}

bool use_pdl() {
    static const bool v = [] {  // read once (thread-safe initialisation)
        const char* e = std::getenv("ABSP_PDL");
        return !(e != nullptr && e[0] == '0');
    }();
    return v;
}

// Device address of a pinned, device-mapped host buffer, else nullptr.
void* mapped_host(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

absp_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
    if (ws == nullptr || !aligned(ws, kAlign)) return ABSP_ERR_INVALID_ARG;
    if (ws_bytes < need) return ABSP_ERR_INVALID_ARG;
    return ABSP_OK;
}

}  // namespace

absp_status absp::check_cent(const absp_centroids* c) {
    if (c == nullptr || c->codes == nullptr) return ABSP_ERR_INVALID_ARG;
    if (c->format != ABSP_CENTROIDS_INT4 && c->format != ABSP_CENTROIDS_BF16)
        return ABSP_ERR_INVALID_ARG;
    if (!aligned(c->codes, kAlign)) return ABSP_ERR_INVALID_ARG;
    if (c->format == ABSP_CENTROIDS_INT4 &&
        (c->scale == nullptr || c->zp == nullptr || !aligned(c->scale, 4) || !aligned(c->zp, 4)))
        return ABSP_ERR_INVALID_ARG;
    return ABSP_OK;
}

namespace {

absp_status run_decode(int mode, const absp_layer_kv* kv, const absp_centroids* cent,
                       const void* q, int32_t budget, int32_t* sel, int32_t* sel_count,
                       void* out, void* ws, size_t ws_bytes, void* stream, uint32_t flags = 0) {
    KvDesc d;
    absp_status st = make_desc(kv, &d, (mode & kModeAttend) != 0);
    if (st != ABSP_OK) return st;
    int32_t kmax = 0, nmax = 0;
    st = check_budget(d, budget, &kmax, &nmax);
    if (st != ABSP_OK) return st;
    if ((mode & kModeSelect) && nmax > ABSP_MAX_BLOCKS_PER_HEAD) return ABSP_ERR_UNSUPPORTED;
    st = check_ws(ws, ws_bytes, kWsHeader);
    if (st != ABSP_OK) return st;
    if (q == nullptr || !aligned(q, 4)) return ABSP_ERR_INVALID_ARG;
    if ((mode & kModeSelect) && (st = check_cent(cent)) != ABSP_OK) return st;
    if (mode == kModeSelect && (sel == nullptr || sel_count == nullptr)) return ABSP_ERR_INVALID_ARG;
    if (mode == kModeAttend && (sel == nullptr || sel_count == nullptr)) return ABSP_ERR_INVALID_ARG;
    if ((mode & kModeAttend) && (out == nullptr || !aligned(out, 4))) return ABSP_ERR_INVALID_ARG;

    CUtensorMap tmk, tmv;
    std::memset(&tmk, 0, sizeof(tmk));
    std::memset(&tmv, 0, sizeof(tmv));
    if (mode & kModeAttend) {
        if ((st = page_tensor_map(d.k_pages, d, &tmk)) != ABSP_OK) return st;
        if ((st = page_tensor_map(d.v_pages, d, &tmv)) != ABSP_OK) return st;
    }
    DecodeArgs a;
    a.kv = d;
    a.codes = cent ? cent->codes : nullptr;
    a.scale = cent ? cent->scale : nullptr;
    a.zp = cent ? cent->zp : nullptr;
    a.cfmt = cent ? cent->format : ABSP_CENTROIDS_INT4;
    a.group_max = (flags & ABSP_STEP_GROUP_MAX) != 0 ? 1 : 0;
    a.diag_timeout = (flags & ABSP_STEP_DIAG_WAIT_TIMEOUT) != 0 ? 1 : 0;
    a.throughput = (flags & ABSP_STEP_THROUGHPUT) != 0 ? 1 : 0;
    if (a.diag_timeout && (mode == kModeAttend || a.group_max || a.cfmt != ABSP_CENTROIDS_INT4 ||
                           d.G > 8 || (flags & ABSP_STEP_EARLY_PREFETCH) != 0))
        return ABSP_ERR_UNSUPPORTED;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.sel = sel;
    a.sel_count = sel_count;
    a.kmax = kmax;
    a.budget = budget;
    a.err = static_cast<int32_t*>(ws);
    a.nmax = nmax;
    const bool early = (flags & ABSP_STEP_EARLY_PREFETCH) != 0;
    return from_cuda(launch_decode(mode, a, &tmk, &tmv, use_pdl(), early,
                                   static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

const char* absp_status_string(absp_status status) {
    switch (status) {
        case ABSP_OK: return "ok";
        case ABSP_ERR_INVALID_ARG: return "invalid argument";
        case ABSP_ERR_UNSUPPORTED: return "unsupported configuration";
        case ABSP_ERR_CUDA: return "CUDA runtime error";
        case ABSP_ERR_DEVICE_FAULT: return "device-side bounds check failed";
        case ABSP_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

absp_status absp_centroid_sizes(const absp_layer_kv* kv, size_t* codes_bytes,
                                size_t* scale_bytes, size_t* zp_bytes) {
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    const size_t params = static_cast<size_t>(d.S) * d.Hkv * ABSP_HEAD_DIM * 4;
    if (codes_bytes) *codes_bytes = static_cast<size_t>(d.S) * d.rows_per_seq * ABSP_CODE_ROW_BYTES;
    if (scale_bytes) *scale_bytes = params;
    if (zp_bytes) *zp_bytes = params;
    return ABSP_OK;
}

absp_status absp_centroid_sizes_fmt(const absp_layer_kv* kv, int32_t format,
                                    size_t* codes_bytes, size_t* scale_bytes, size_t* zp_bytes) {
    if (format != ABSP_CENTROIDS_INT4 && format != ABSP_CENTROIDS_BF16) return ABSP_ERR_INVALID_ARG;
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    const bool bf = format == ABSP_CENTROIDS_BF16;
    const size_t params = bf ? 0 : static_cast<size_t>(d.S) * d.Hkv * ABSP_HEAD_DIM * 4;
    if (codes_bytes)
        *codes_bytes = static_cast<size_t>(d.S) * d.rows_per_seq * (bf ? 2 * ABSP_HEAD_DIM
                                                                      : ABSP_CODE_ROW_BYTES);
    if (scale_bytes) *scale_bytes = params;
    if (zp_bytes) *zp_bytes = params;
    return ABSP_OK;
}

absp_status absp_centroid_row_offset(const absp_layer_kv* kv, int32_t seq, int32_t kv_head,
                                     int64_t* row) {
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if (row == nullptr || seq < 0 || seq >= d.S || kv_head < 0 || kv_head >= d.Hkv)
        return ABSP_ERR_INVALID_ARG;
    *row = static_cast<int64_t>(seq) * d.rows_per_seq + d.row_base[kv_head];
    return ABSP_OK;
}

absp_status absp_build_workspace_size(const absp_layer_kv* kv, size_t* bytes) {
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if (bytes == nullptr) return ABSP_ERR_INVALID_ARG;
    *bytes = build_ws_bytes(d);
    return ABSP_OK;
}

absp_status absp_decode_workspace_size(const absp_layer_kv* kv, int32_t budget_tokens,
                                       size_t* bytes) {
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if ((st = check_budget(d, budget_tokens, nullptr, nullptr)) != ABSP_OK) return st;
    if (bytes == nullptr) return ABSP_ERR_INVALID_ARG;
    *bytes = decode_ws_bytes(d);
    return ABSP_OK;
}

absp_status absp_select_capacity(const absp_layer_kv* kv, int32_t budget_tokens, int32_t* kmax) {
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if (kmax == nullptr) return ABSP_ERR_INVALID_ARG;
    return check_budget(d, budget_tokens, kmax, nullptr);
}

absp_status absp_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    ABSP_TRACE("absp_workspace_init");
    if (ws == nullptr || ws_bytes < static_cast<size_t>(kWsHeader) || !aligned(ws, kAlign))
        return ABSP_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

absp_status absp_build_centroids(const absp_layer_kv* kv, void* ws, size_t ws_bytes, void* stream) {
    ABSP_TRACE("absp_build_centroids");
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if ((st = check_ws(ws, ws_bytes, build_ws_bytes(d))) != ABSP_OK) return st;
    return from_cuda(launch_build(d, build_ws_layout(ws, d), static_cast<cudaStream_t>(stream)));
}

absp_status absp_quantize_centroids(const absp_layer_kv* kv, void* ws, size_t ws_bytes,
                                    const absp_centroids* out, void* stream) {
    ABSP_TRACE("absp_quantize_centroids");
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if ((st = check_ws(ws, ws_bytes, build_ws_bytes(d))) != ABSP_OK) return st;
    if ((st = check_cent(out)) != ABSP_OK) return st;
    return from_cuda(launch_quantize(d, build_ws_layout(ws, d), out->codes, out->scale, out->zp,
                                     out->format, static_cast<cudaStream_t>(stream)));
}

absp_status absp_build_quantize_centroids(const absp_layer_kv* kv, void* ws, size_t ws_bytes,
                                          const absp_centroids* out, void* stream) {
    ABSP_TRACE("absp_build_quantize_centroids");
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if ((st = check_ws(ws, ws_bytes, build_ws_bytes(d))) != ABSP_OK) return st;
    if ((st = check_cent(out)) != ABSP_OK) return st;
    return from_cuda(launch_build_quantize(d, build_ws_layout(ws, d), out->codes, out->scale,
                                           out->zp, out->format,
                                           static_cast<cudaStream_t>(stream)));
}

absp_status absp_append_centroids(const absp_layer_kv* kv, const absp_centroids* cent,
                                  int32_t* exceeded, void* ws, size_t ws_bytes, void* stream) {
    ABSP_TRACE("absp_append_centroids");
    KvDesc d;
    absp_status st = make_desc(kv, &d, false);
    if (st != ABSP_OK) return st;
    if ((st = check_cent(cent)) != ABSP_OK) return st;
    if ((st = check_ws(ws, ws_bytes, kWsHeader)) != ABSP_OK) return st;
    if (exceeded != nullptr && !aligned(exceeded, 4)) return ABSP_ERR_INVALID_ARG;
    return from_cuda(launch_append(d, cent->codes, cent->scale, cent->zp, cent->format, exceeded,
                                   static_cast<int32_t*>(ws), static_cast<cudaStream_t>(stream)));
}

absp_status absp_score_select(const absp_layer_kv* kv, const absp_centroids* cent, const void* q,
                              int32_t budget_tokens, int32_t* sel, int32_t* sel_count, void* ws,
                              size_t ws_bytes, void* stream) {
    ABSP_TRACE("absp_score_select");
    return run_decode(kModeSelect, kv, cent, q, budget_tokens, sel, sel_count, nullptr, ws,
                      ws_bytes, stream);
}

absp_status absp_sparse_decode(const absp_layer_kv* kv, const void* q, const int32_t* sel,
                               const int32_t* sel_count, int32_t budget_tokens, void* out,
                               void* ws, size_t ws_bytes, void* stream) {
    ABSP_TRACE("absp_sparse_decode");
    return run_decode(kModeAttend, kv, nullptr, q, budget_tokens, const_cast<int32_t*>(sel),
                      const_cast<int32_t*>(sel_count), out, ws, ws_bytes, stream);
}

absp_status absp_decode_step(const absp_layer_kv* kv, const absp_centroids* cent, const void* q,
                             int32_t budget_tokens, void* out, void* ws, size_t ws_bytes,
                             void* stream) {
    ABSP_TRACE("absp_decode_step");
    return run_decode(kModeFull, kv, cent, q, budget_tokens, nullptr, nullptr, out, ws, ws_bytes,
                      stream);
}

absp_status absp_decode_step_ex(const absp_layer_kv* kv, const absp_centroids* cent,
                                const void* q, int32_t budget_tokens, void* out, void* ws,
                                size_t ws_bytes, uint32_t flags, void* stream) {
    ABSP_TRACE("absp_decode_step_ex");
    if ((flags & ~static_cast<uint32_t>(ABSP_STEP_EARLY_PREFETCH | ABSP_STEP_GROUP_MAX |
                                        ABSP_STEP_THROUGHPUT | ABSP_STEP_DIAG_WAIT_TIMEOUT)) != 0)
        return ABSP_ERR_INVALID_ARG;
    return run_decode(kModeFull, kv, cent, q, budget_tokens, nullptr, nullptr, out, ws, ws_bytes,
                      stream, flags);
}

absp_status absp_score_select_ex(const absp_layer_kv* kv, const absp_centroids* cent, const void* q,
                                 int32_t budget_tokens, int32_t* sel, int32_t* sel_count,
                                 void* ws, size_t ws_bytes, uint32_t flags, void* stream) {
    ABSP_TRACE("absp_score_select_ex");
    if ((flags & ~static_cast<uint32_t>(ABSP_STEP_GROUP_MAX | ABSP_STEP_DIAG_WAIT_TIMEOUT)) != 0)
        return ABSP_ERR_INVALID_ARG;
    return run_decode(kModeSelect, kv, cent, q, budget_tokens, sel, sel_count, nullptr, ws,
                      ws_bytes, stream, flags);
}

absp_status absp_decode_step_host(const absp_layer_kv* kv, const absp_centroids* cent,
                                  const void* q_host, int32_t budget_tokens, void* out_host,
                                  void* ws, size_t ws_bytes, void* stream) {
    ABSP_TRACE("absp_decode_step_host");
    return absp_decode_step_host_ex(kv, cent, q_host, budget_tokens, out_host, ws, ws_bytes, 0,
                                    stream);
}

absp_status absp_decode_step_host_ex(const absp_layer_kv* kv, const absp_centroids* cent,
                                     const void* q_host, int32_t budget_tokens, void* out_host,
                                     void* ws, size_t ws_bytes, uint32_t flags, void* stream) {
    ABSP_TRACE("absp_decode_step_host_ex");
    if ((flags & ~static_cast<uint32_t>(ABSP_STEP_EARLY_PREFETCH | ABSP_STEP_GROUP_MAX)) != 0)
        return ABSP_ERR_INVALID_ARG;
    KvDesc d;
    absp_status st = make_desc(kv, &d, true);
    if (st != ABSP_OK) return st;
    if ((st = check_ws(ws, ws_bytes, decode_ws_bytes(d))) != ABSP_OK) return st;
    if (q_host == nullptr || out_host == nullptr) return ABSP_ERR_INVALID_ARG;
    // pinned host buffers mapped into the device address space: the kernel
    // reads the query and writes the output across the host link itself
    void* qm = mapped_host(q_host);
    void* om = mapped_host(out_host);
    if (qm != nullptr && om != nullptr && aligned(qm, 4) && aligned(om, 4))
        return run_decode(kModeFull, kv, cent, qm, budget_tokens, nullptr, nullptr, om, ws,
                          ws_bytes, stream, flags);
    const size_t act = static_cast<size_t>(d.S) * d.Hq * ABSP_HEAD_DIM * 2;
    uint8_t* qd = static_cast<uint8_t*>(ws) + kWsHeader;
    uint8_t* od = qd + round_up(act, kAlign);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(qd, q_host, act, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return from_cuda(e);
    st = run_decode(kModeFull, kv, cent, qd, budget_tokens, nullptr, nullptr, od, ws, ws_bytes,
                    stream, flags);
    if (st != ABSP_OK) return st;
    e = cudaMemcpyAsync(out_host, od, act, cudaMemcpyDeviceToHost, s);
    return from_cuda(e);
}

absp_status absp_check_device_error(void* ws, size_t ws_bytes, void* stream, int32_t* detail) {
    ABSP_TRACE("absp_check_device_error");
    if (ws == nullptr || ws_bytes < static_cast<size_t>(kWsHeader)) return ABSP_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t word[2] = {0, 0};
    cudaError_t e = cudaMemcpyAsync(word, ws, sizeof(word), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return from_cuda(e);
    if (detail) *detail = word[1];
    if (word[0] == 0) return ABSP_OK;
    e = cudaMemsetAsync(ws, 0, sizeof(word), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return from_cuda(e);
    return word[0] == ABSP_ERR_TIMEOUT ? ABSP_ERR_TIMEOUT : ABSP_ERR_DEVICE_FAULT;
}

#ifndef ABSP_BUILD_ID
#define ABSP_BUILD_ID "unknown"
#endif

const char* absp_build_id(void) { return ABSP_BUILD_ID; }

int absp_last_cuda_error(void) { return t_last_cuda; }

const char* absp_last_cuda_error_string(void) {
    return t_last_cuda == 0 ? "no error" : cudaGetErrorString(static_cast<cudaError_t>(t_last_cuda));
}

}  // extern "C"
