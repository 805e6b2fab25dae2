// Internal declarations shared by the libabsp translation units: the
// by-value layer descriptor handed to every kernel, small PTX wrappers
// (mbarrier, bulk / tensor copies, cluster barriers and distributed shared
// memory, programmatic dependent launch, ldmatrix, mma) and the launchers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "absp.h"

namespace absp {

constexpr int kD = ABSP_HEAD_DIM;        // channels per head
constexpr int kPage = ABSP_PAGE_SIZE;    // tokens per physical page
constexpr int kRowBytes = ABSP_CODE_ROW_BYTES;
constexpr int kWsHeader = 256;           // error word + detail, padded

// Everything a kernel needs to address one layer.  Passed by value.
struct KvDesc {
    int32_t S, Hq, Hkv, G;
    int32_t max_pages;
    int32_t pad_;
    int64_t num_phys_pages;
    int64_t rows_per_seq;                // code rows per sequence (all heads)
    const int32_t* seq_lens;
    const int32_t* page_table;
    const __nv_bfloat16* k_pages;
    const __nv_bfloat16* v_pages;
    int32_t bs[ABSP_MAX_KV_HEADS];       // block size per KV head
    int32_t row_base[ABSP_MAX_KV_HEADS]; // first code row of each head
    int32_t cap[ABSP_MAX_KV_HEADS];      // code-row capacity of each head
};

// ---------------------------------------------------------------- errors --

__device__ __forceinline__ void set_error(int32_t* err, int code, int detail) {
    if (atomicCAS(err, 0, code) == 0) atomicExch(err + 1, detail);
}

// -------------------------------------------------------------- helpers --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ----------------------------------------------------------- mbarriers --

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Same wait with cluster-scope acquire: orders the distributed-shared-memory
// writes of the CTAs that arrived remotely before reads that follow.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Arrive (release, cluster scope) on an mbarrier of another CTA of the
// cluster; `remote` is a shared::cluster address from dsmem_addr().
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote)
                 : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Bulk prefetch of `bytes` (a multiple of 16; p 16-byte aligned) into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Default limit of a bounded device wait.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// Wait for phase `parity` of an mbarrier, giving up after `limit_ns`.  On
// timeout the error word records ABSP_ERR_TIMEOUT (detail = `where`) and the
// caller carries on (so that every later cluster barrier is still reached);
// results are then garbage and the host sees the error.
template <bool CLUSTER_ACQUIRE = false>
__device__ __forceinline__ void mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  int32_t* err, int where,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    auto poll = [&] {
        return CLUSTER_ACQUIRE ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    };
    if (poll()) return;
    const uint64_t t0 = globaltimer_ns();
    while (!poll()) {
        if (globaltimer_ns() - t0 > limit_ns) {
            set_error(err, ABSP_ERR_TIMEOUT, where);
            return;
        }
    }
}

// ------------------------------------------------------- async copies --

// 4-byte asynchronous copy global -> shared (no register staging); completed
// by cp_async_wait_all() in the issuing thread.
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// 1-D bulk copy global -> this CTA's shared memory; completes `bytes` of
// transaction count on `bar`.  16-byte aligned addresses, size % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Fetch a tensor-map descriptor (a __grid_constant__ kernel parameter) into
// the copy engine's descriptor cache ahead of its first use.
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tensor tile load into this CTA's own shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x,
                                            int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// ------------------------------------------------------------ clusters --

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t dsmem_addr(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

// Asynchronous 16-byte store into a CTA of the cluster that completes 16
// bytes of transaction count on that CTA's mbarrier `remote_bar` (both
// shared::cluster addresses of the same destination CTA).
__device__ __forceinline__ void st_async_v4(uint32_t remote_addr, float a, float b, float c,
                                            float d, uint32_t remote_bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, "
        "[%5];" ::"r"(remote_addr),
        "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
        : "memory");
}

// 8-byte variant of st_async_v4.
__device__ __forceinline__ void st_async_v2(uint32_t remote_addr, float a, float b,
                                            uint32_t remote_bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
            remote_addr),
        "f"(a), "f"(b), "r"(remote_bar)
        : "memory");
}

__device__ __forceinline__ void dsmem_st_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ int32_t dsmem_ld_s32(uint32_t addr) {
    int32_t v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// ------------------------------------------- programmatic dependent launch --

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------- warp matrix ops --

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                        uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16(float& d0, float& d1, float& d2, float& d3,
                                         uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

#pragma nv_diag_suppress 550  // the discarded rows 8..15 below
// Same tile op when rows 8..15 of A are zero (a GQA group of <= 8 heads):
// only the accumulators of rows 0..7 are carried; rows 8..15 are written to
// discarded temporaries and read as zero.
__device__ __forceinline__ void mma_bf16_top(float& d0, float& d1, uint32_t a0, uint32_t a2,
                                             uint32_t b0, uint32_t b1) {
    float x2, x3;  // rows 8..15: discarded
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %12};"
        : "=f"(d0), "=f"(d1), "=f"(x2), "=f"(x3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0), "f"(d1), "f"(0.0f));
}
#pragma nv_diag_default 550

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ----------------------------------------------------- host validation --

// Checks a layer description and fills the kernel descriptor (abi.cu).
absp_status make_desc(const absp_layer_kv* kv, KvDesc* d, bool need_v);
// ABSP_OK for cudaSuccess; otherwise records `e` as the calling thread's last
// CUDA error (absp_last_cuda_error) and returns ABSP_ERR_CUDA.
absp_status cuda_status(int e);
// Checks the three centroid buffers (abi.cu).
absp_status check_cent(const absp_centroids* c);

// ------------------------------------------------------------ launchers --

// Build step (centroids.cu)
struct BuildWs {
    int32_t* err;
    unsigned long long* minmax;   // mins [S][Hkv][128], then mins of the negated values
                                  // (= -max), order-mapped fp64 keys
    double* cent;                 // [S][rows_per_seq][128]
};
BuildWs build_ws_layout(void* ws, const KvDesc& kv);
size_t build_ws_bytes(const KvDesc& kv);
cudaError_t launch_build(const KvDesc& kv, const BuildWs& w, cudaStream_t st);
// format: ABSP_CENTROIDS_INT4 (codes + scale + zp) or ABSP_CENTROIDS_BF16
cudaError_t launch_quantize(const KvDesc& kv, const BuildWs& w, uint8_t* codes, float* scale,
                            int32_t* zp, int format, cudaStream_t st);

// Steps 1-2 in one call (centroids.cu): the build kernel and the quantise
// kernel (INT4), or the build kernel writing bf16 rows directly (BF16).
cudaError_t launch_build_quantize(const KvDesc& kv, const BuildWs& w, uint8_t* codes, float* scale,
                                  int32_t* zp, int format, cudaStream_t st);

// Incremental tail-row update after appended tokens (centroids.cu)
cudaError_t launch_append(const KvDesc& kv, uint8_t* codes, const float* scale, const int32_t* zp,
                          int format, int32_t* exceeded, int32_t* err, cudaStream_t st);

// Decode steps (decode.cu)
enum DecodeMode : int { kModeSelect = 1, kModeAttend = 2, kModeFull = 3 };

struct DecodeArgs {
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
    int32_t nmax;                 // bound on blocks per head for this layer
    int32_t cfmt;                 // centroid format (ABSP_CENTROIDS_*)
    int32_t group_max;            // score = max over the GQA group's heads
    int32_t diag_timeout;         // ABSP_STEP_DIAG_WAIT_TIMEOUT: the failure-path diagnostic
    int32_t throughput;           // ABSP_STEP_THROUGHPUT: half as many CTAs per head
};
// early_prefetch: codes, parameters, lengths and page table are read before
// the programmatic-dependency wait (only the query after it).
cudaError_t launch_decode(int mode, const DecodeArgs& a, const CUtensorMap* tmk,
                          const CUtensorMap* tmv, bool pdl, bool early_prefetch, cudaStream_t st);

}  // namespace absp
