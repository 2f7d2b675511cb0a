// C-ABI of the dllm_qgemm library (see include/dllm_qgemm.h for the contract).
#include <cstdio>
#include <cstring>

#include "../../include/dllm_qgemm.h"
#include "layout.cuh"
#include "qgemm.cuh"

using namespace dllm;

namespace {

constexpr int MAX_DEV = 64;
int g_dev_checked[MAX_DEV];  // 0 unknown, 1 sm_100, -1 other
int g_num_sms[MAX_DEV];
bool g_attr_done[MAX_DEV][4];

int current_device(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= MAX_DEV) return DLLM_ERR_CUDA;
    if (g_dev_checked[*dev] == 0) {
        cudaDeviceProp p;
        if (cudaGetDeviceProperties(&p, *dev) != cudaSuccess) return DLLM_ERR_CUDA;
        g_dev_checked[*dev] = (p.major == 10 && p.minor == 0) ? 1 : -1;
        g_num_sms[*dev] = p.multiProcessorCount;
    }
    return g_dev_checked[*dev] == 1 ? DLLM_OK : DLLM_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA;
}

int grid_for(int64_t work, int64_t per_block) {
    int64_t g = (work + per_block - 1) / per_block;
    if (g > 65535LL * 32) g = 65535LL * 32;
    return (int)(g < 1 ? 1 : g);
}

template <int QT, bool DBG>
int run_gemm(GemmArgs& a, cudaStream_t s) {
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    constexpr size_t smem = gemm_smem_bytes<QT>();
    const int slot = (QT == 12 ? 0 : 2) + (DBG ? 1 : 0);
    if (!g_attr_done[dev][slot]) {
        if (cudaFuncSetAttribute(qgemm_kernel<QT, DBG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return DLLM_ERR_CUDA;
        g_attr_done[dev][slot] = true;
    }
    const int64_t rows_total = a.rows ? round_up(a.n_rows, 16) : a.Mp;
    a.n_st = (int32_t)((rows_total + UNIT_TOKENS - 1) / UNIT_TOKENS);
    a.mu = (int32_t)round_up((rows_total + a.n_st - 1) / a.n_st, 16);
    const int64_t units = (int64_t)a.n_tiles * a.n_st;
    const int grid = (int)(units < g_num_sms[dev] ? units : g_num_sms[dev]);
    qgemm_kernel<QT, DBG><<<grid, GEMM_THREADS, smem, s>>>(a);
    return launch_status();
}

int check_shape(dllm_qtype t, int64_t N, int64_t K) {
    if (t != DLLM_Q4_K && t != DLLM_Q6_K) return DLLM_ERR_ARG;
    if (N <= 0 || K <= 0 || N % TROWS || K % QK) return DLLM_ERR_ARG;
    if (N / TROWS > (1LL << 30) || K / QK > (1 << 20)) return DLLM_ERR_ARG;
    return DLLM_OK;
}

int check_act(const int8_t* q, const float* scale, const uint8_t* sums, int64_t M) {
    if (!q || !scale || !sums || M <= 0) return DLLM_ERR_ARG;
    if (!aligned16(q) || !aligned16(scale) || !aligned16(sums)) return DLLM_ERR_ALIGN;
    return DLLM_OK;
}

}  // namespace

extern "C" {

int dllm_repacked_bytes(dllm_qtype t, int64_t N, int64_t K, size_t* out_bytes) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if (!out_bytes) return DLLM_ERR_ARG;
    *out_bytes = (size_t)N * (size_t)(K / QK) * (t == DLLM_Q4_K ? Q4K_BLOCK : Q6K_BLOCK);
    return DLLM_OK;
}

static int repack(dllm_qtype t, const void* src, int64_t N, int64_t K, void* dst, dllm_stream_t stream) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if (!src || !dst) return DLLM_ERR_ARG;
    if (!aligned16(dst)) return DLLM_ERR_ALIGN;
    const size_t bytes = (size_t)N * (K / QK) * (t == DLLM_Q4_K ? Q4K_BLOCK : Q6K_BLOCK);
    const uint8_t* s8 = static_cast<const uint8_t*>(src);
    const uint8_t* d8 = static_cast<const uint8_t*>(dst);
    if (s8 < d8 + bytes && d8 < s8 + bytes) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t chunks = (int64_t)(bytes / 16);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (t == DLLM_Q4_K)
        repack_q4k_kernel<<<grid_for(chunks, 256), 256, 0, s>>>(s8, N, K / QK, static_cast<uint8_t*>(dst));
    else
        repack_q6k_kernel<<<grid_for(chunks, 256), 256, 0, s>>>(s8, N, K / QK, static_cast<uint8_t*>(dst));
    return launch_status();
}

int dllm_repack_q4k(const void* g, int64_t N, int64_t K, void* dst, dllm_stream_t s) {
    return repack(DLLM_Q4_K, g, N, K, dst, s);
}
int dllm_repack_q6k(const void* g, int64_t N, int64_t K, void* dst, dllm_stream_t s) {
    return repack(DLLM_Q6_K, g, N, K, dst, s);
}

int dllm_act_bytes(int64_t M, int64_t K, size_t* q_bytes, size_t* scale_bytes, size_t* sums_bytes) {
    if (M <= 0 || K <= 0 || K % QK || !q_bytes || !scale_bytes || !sums_bytes) return DLLM_ERR_ARG;
    const int64_t Mp = round_up(M, 16);
    *q_bytes = (size_t)Mp * K;
    *scale_bytes = (size_t)Mp * (K / QK) * 4;
    *sums_bytes = (size_t)Mp * (K / QK) * 16;
    return DLLM_OK;
}

int dllm_quantize_act(const float* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* scale, uint8_t* sums,
                      dllm_stream_t stream) {
    if (!x || M <= 0 || K <= 0 || K % QK || ldx < K) return DLLM_ERR_ARG;
    int rc = check_act(q, scale, sums, M);
    if (rc) return rc;
    if (!aligned16(x) || ldx % 4) return DLLM_ERR_ALIGN;
    if (M > (1LL << 31) || K / QK > 65535) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t Mp = round_up(M, 16);
    dim3 grid((unsigned)(Mp / 8), (unsigned)(K / QK));
    quantize_act_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, M, ldx, Mp, q, scale, sums);
    return launch_status();
}

int dllm_qgemm_workspace_bytes(dllm_qtype t, int64_t N, int64_t K, int64_t M, size_t* bytes) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if (M <= 0 || !bytes) return DLLM_ERR_ARG;
    *bytes = 0;  // the current schedule needs no scratch
    return DLLM_OK;
}

static int gemm_common(GemmArgs& a, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
                       const uint8_t* sums, int64_t M, const int32_t* rows, int64_t n_rows) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if ((rc = check_act(q, scale, sums, M))) return rc;
    if (rows && (n_rows < 1 || n_rows > 32)) return DLLM_ERR_ARG;
    if (M > (1LL << 31)) return DLLM_ERR_ARG;
    memset(&a, 0, sizeof(a));
    a.nsb = (int32_t)(K / QK);
    a.q = q;
    a.scale = scale;
    a.sums = sums;
    a.M = M;
    a.Mp = round_up(M, 16);
    a.rows = rows;
    a.n_rows = rows ? (int32_t)n_rows : 0;
    a.m_out = rows ? n_rows : M;
    return DLLM_OK;
}

static int dispatch(GemmArgs& a, dllm_qtype t, bool dbg, dllm_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (t == DLLM_Q4_K) return dbg ? run_gemm<12, true>(a, s) : run_gemm<12, false>(a, s);
    return dbg ? run_gemm<14, true>(a, s) : run_gemm<14, false>(a, s);
}

int dllm_qgemm(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
               const uint8_t* sums, int64_t M, const int32_t* rows, int64_t n_rows, float* out, int64_t ldo,
               void* workspace, size_t workspace_bytes, dllm_stream_t stream) {
    (void)workspace;
    (void)workspace_bytes;
    GemmArgs a;
    int rc = gemm_common(a, t, N, K, q, scale, sums, M, rows, n_rows);
    if (rc) return rc;
    if (!w || !out || ldo < N) return DLLM_ERR_ARG;
    if (!aligned16(w) || !aligned16(out) || ldo % 4) return DLLM_ERR_ALIGN;
    if (rows && !aligned16(rows)) return DLLM_ERR_ALIGN;
    a.seg[0] = Segment{static_cast<const uint8_t*>(w), out, ldo, 0};
    a.nseg = 1;
    a.n_tiles = (int32_t)(N / TROWS);
    return dispatch(a, t, false, stream);
}

int dllm_qkv_qgemm(const void* wq, const void* wk, const void* wv, dllm_qtype t, int64_t Nq, int64_t Nkv, int64_t K,
                   const int8_t* q, const float* scale, const uint8_t* sums, int64_t M, float* oq, int64_t ldo_q,
                   float* ok, float* ov, int64_t ldo_kv, void* workspace, size_t workspace_bytes,
                   dllm_stream_t stream) {
    (void)workspace;
    (void)workspace_bytes;
    GemmArgs a;
    int rc = gemm_common(a, t, Nq, K, q, scale, sums, M, nullptr, 0);
    if (rc) return rc;
    if ((rc = check_shape(t, Nkv, K))) return rc;
    if (!wq || !wk || !oq || !ok || (wv && !ov) || ldo_q < Nq || ldo_kv < Nkv) return DLLM_ERR_ARG;
    if (!aligned16(wq) || !aligned16(wk) || (wv && !aligned16(wv)) || !aligned16(oq) || !aligned16(ok) ||
        (wv && !aligned16(ov)) || ldo_q % 4 || ldo_kv % 4)
        return DLLM_ERR_ALIGN;
    const int32_t tq = (int32_t)(Nq / TROWS), tkv = (int32_t)(Nkv / TROWS);
    a.seg[0] = Segment{static_cast<const uint8_t*>(wq), oq, ldo_q, 0};
    a.seg[1] = Segment{static_cast<const uint8_t*>(wk), ok, ldo_kv, tq};
    a.nseg = 2;
    a.n_tiles = tq + tkv;
    if (wv) {
        a.seg[2] = Segment{static_cast<const uint8_t*>(wv), ov, ldo_kv, tq + tkv};
        a.nseg = 3;
        a.n_tiles += tkv;
    }
    return dispatch(a, t, false, stream);
}

int dllm_get_device_status(dllm_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return DLLM_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof(int)) != cudaSuccess) return DLLM_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_err, &zero, sizeof(int)) != cudaSuccess) return DLLM_ERR_CUDA;
    return v;
}

const char* dllm_status_string(int code) {
    switch (code) {
        case DLLM_OK: return "ok";
        case DLLM_ERR_ARG: return "invalid argument";
        case DLLM_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
        case DLLM_ERR_UNSUPPORTED: return "device is not sm_100";
        case DLLM_ERR_CUDA: return "CUDA runtime error";
        case DLLM_ERR_ROW_RANGE: return "row index out of range";
        case DLLM_ERR_TIMEOUT: return "bounded device wait ran out";
        case DLLM_ERR_WORKSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

// ---------------------------------------------------------------- test-only kernels

}  // extern "C"

namespace dllm {

// Per-sub-block integer dots straight from the repacked tiles and the tiled
// activations, on CUDA cores.  One thread per (m, n, super-block).
__global__ void subblock_dots_kernel(const uint8_t* __restrict__ w, int qt, int64_t N, int nsb,
                                     const int8_t* __restrict__ q, int64_t M, int64_t Mp, int32_t* __restrict__ dots) {
    const int64_t total = M * N * nsb;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
        const int s = (int)(g % nsb);
        const int64_t n = (g / nsb) % N;
        const int64_t m = g / nsb / N;
        const int64_t t = n / TROWS;
        const int r = (int)(n % TROWS);
        auto act = [&](int k) -> int {  // k within the super-block
            return q[(((int64_t)s * (Mp / 8) + m / 8) * 16 + k / 16) * 128 + (m % 8) * 16 + (k % 16)];
        };
        if (qt == 12) {
            const uint8_t* tl = w + (t * nsb + s) * (int64_t)Q4K_TILE;
            for (int j = 0; j < 8; j++) {
                int acc = 0;
                for (int l = 0; l < 32; l++) {
                    const int byte = 32 * (j / 2) + l;  // quant byte within the row
                    const uint8_t b = tl[((byte / 16) * TROWS + r) * 16 + byte % 16];
                    const int qv = (j & 1) ? (b >> 4) : (b & 15);
                    acc += qv * act(32 * j + l);
                }
                dots[(m * N + n) * (8LL * nsb) + 8 * s + j] = acc;
            }
        } else {
            const uint8_t* tl = w + (t * nsb + s) * (int64_t)Q6K_TILE;
            for (int j = 0; j < 16; j++) {
                int acc = 0;
                for (int l = 0; l < 16; l++) {
                    const int k = 16 * j + l;
                    const int h = k / 128, e = k % 128, gg = e / 32, ll = e % 32;
                    const int lb = 64 * h + ll + 32 * (gg & 1);
                    const uint8_t lo = tl[((lb / 16) * TROWS + r) * 16 + lb % 16];
                    const int hb = 32 * h + ll;
                    const uint8_t hi = tl[Q6K_OFF_QH + ((hb / 16) * TROWS + r) * 16 + hb % 16];
                    const int qv = ((gg < 2) ? (lo & 15) : (lo >> 4)) | (((hi >> (2 * gg)) & 3) << 4);
                    acc += (qv - 32) * act(k);
                }
                dots[(m * N + n) * (16LL * nsb) + 16 * s + j] = acc;
            }
        }
    }
}

// Back-to-back 128 x n x 32 int8 MMAs, B in shared memory, A in tensor memory
// (a_tmem != 0) or shared memory, rotating over n_acc independent accumulators.
__global__ void __launch_bounds__(128, 1) bench_mma_kernel(int n, int n_acc, int a_tmem, int iters,
                                                           unsigned long long* ns_out) {
    extern __shared__ __align__(1024) uint8_t bsm[];
    __shared__ uint32_t tbase;
    __shared__ __align__(8) uint64_t bar;
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (256 * 32 + 128 * 32) / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(bsm)[i] = 0x01010101u;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(&tbase, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tbase;
    if (threadIdx.x == 0) {
        const uint32_t id = idesc_i8(128, n, 0, 1);
        const uint64_t bd = sdesc_kmajor_noswz(smem_u32(bsm), 128, 256);
        const uint64_t ad = sdesc_kmajor_noswz(smem_u32(bsm + 256 * 32), 128, 256);
        const uint64_t t0 = globaltimer_ns();
        for (int i = 0; i < iters; i++) {
            const uint32_t d = tm + (uint32_t)((i % n_acc) * n);
            if (a_tmem)
                mma_i8_ts(d, tm + 448 + 8 * (i & 7), bd, id, i >= n_acc);
            else
                mma_i8_ss(d, ad, bd, id, i >= n_acc);
        }
        tc_commit(&bar);
        uint64_t tw = globaltimer_ns();
        while (!mbar_try_wait(&bar, 0)) {
            if (globaltimer_ns() - tw > WAIT_LIMIT_NS) { set_err(ERR_TIMEOUT); break; }
        }
        ns_out[blockIdx.x] = globaltimer_ns() - t0;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

}  // namespace dllm

extern "C" {

int dllm_debug_subblock_dots(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, int64_t M,
                             int32_t* dots, dllm_stream_t stream) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if (!w || !q || !dots || M <= 0) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t work = M * N * (K / QK);
    subblock_dots_kernel<<<grid_for(work, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(w), (int)t, N, (int)(K / QK), q, M, round_up(M, 16), dots);
    return launch_status();
}

int dllm_debug_sb_ints(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
                       const uint8_t* sums, int64_t M, int32_t* S, int32_t* Smin, dllm_stream_t stream) {
    GemmArgs a;
    int rc = gemm_common(a, t, N, K, q, scale, sums, M, nullptr, 0);
    if (rc) return rc;
    if (!w || !S || (t == DLLM_Q4_K && !Smin)) return DLLM_ERR_ARG;
    a.seg[0] = Segment{static_cast<const uint8_t*>(w), nullptr, N, 0};
    a.nseg = 1;
    a.n_tiles = (int32_t)(N / TROWS);
    a.dbg_S = S;
    a.dbg_Smin = Smin;
    a.dbg_N = N;
    return dispatch(a, t, true, stream);
}

int dllm_bench_mma_i8(int n, int n_acc, int a_from_tmem, int iters, int ctas, unsigned long long* ns_out,
                      dllm_stream_t stream) {
    if (n < 16 || n > 256 || n % 16 || n_acc < 1 || n * n_acc > 448 || iters < 1 || ctas < 1 || ctas > 4096 ||
        !ns_out)
        return DLLM_ERR_ARG;
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    const int smem = 120 * 1024;  // also keeps one CTA per SM
    if (cudaFuncSetAttribute(bench_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return DLLM_ERR_CUDA;
    bench_mma_kernel<<<ctas, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(n, n_acc, a_from_tmem, iters,
                                                                                  ns_out);
    return launch_status();
}

}  // extern "C"
