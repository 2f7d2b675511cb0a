// C-ABI of the dllm_qgemm library (see include/dllm_qgemm.h for the contract).
#include <cstdio>
#include <cstring>

#include "../../include/dllm_qgemm.h"
#include "actfuse.cuh"
#include "attention.cuh"
#include "q80.cuh"
#include "layout.cuh"
#include "qgemm.cuh"

using namespace dllm;

namespace {

constexpr int MAX_DEV = 64;
int g_dev_checked[MAX_DEV];  // 0 unknown, 1 sm_100, -1 other
int g_num_sms[MAX_DEV];
bool g_attr_done[MAX_DEV][8];
bool g_att_attr_done[MAX_DEV];

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

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel on the stream finishes, and synchronises with it on the device
// (pdl_wait) before touching memory that kernel can write.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (the
// library does not link the driver API).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static const EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// A [rows][heads][128] f16 tensor as the 3-D tensor (head dim, head, row) with boxes of
// 64 head-dim values x 1 head x box_rows rows, 128-byte swizzled (half a tile).
bool encode_head_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t heads, int box_rows) {
    const EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)ATT_DH, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)ATT_DH * 2, (cuuint64_t)(heads * ATT_DH * 2)};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The last few encoded maps, per host thread (a layer's q, k and v, a few layers deep):
// encoding costs about as much host time as the launch itself.
bool cached_head_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t heads, int box_rows) {
    struct Entry {
        const void* base;
        int64_t rows, heads;
        int box_rows;
        CUtensorMap map;
    };
    constexpr int N = 12;
    thread_local Entry cache[N] = {};
    thread_local int next = 0;
    for (int i = 0; i < N; i++)
        if (cache[i].base == base && cache[i].rows == rows && cache[i].heads == heads &&
            cache[i].box_rows == box_rows) {
            *m = cache[i].map;
            return true;
        }
    if (!encode_head_rows(m, base, rows, heads, box_rows)) return false;
    cache[next] = {base, rows, heads, box_rows, *m};
    next = (next + 1) % N;
    return true;
}

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA;
}

int grid_for(int64_t work, int64_t per_block) {
    int64_t g = (work + per_block - 1) / per_block;
    if (g > 65535LL * 32) g = 65535LL * 32;
    return (int)(g < 1 ? 1 : g);
}

// K-chunks per tile.  A function of the tile count, the super-block count and the
// SM count only (never of M or of a row list), so that every call on the same
// weight shape sums the same partials in the same order.  Cost model, in units of
// one super-block of one tile, fitted to measured launch times at 128 canvas rows:
// the busiest SM runs ceil(units / SMs) work units, each costing its super-blocks
// plus 2.35 for the unit's start and drain, plus 2.7 more when the tile's K range is
// split (partial write, arrival counter, and the last arriver's chunk sum); chunks
// are at least 4 super-blocks long.
int choose_kc(int64_t n_tiles, int64_t nsb, int sms) {
    int best = 1;
    int64_t best_cost = -1;
    for (int kc = 1; kc <= MAX_KC && kc <= nsb; kc++) {
        const int64_t len = (nsb + kc - 1) / kc;
        if (kc > 1 && len < 4) break;
        const int64_t per_sm = (n_tiles * kc + sms - 1) / sms;
        const int64_t cost = per_sm * (100 * len + 235 + (kc > 1 ? 270 : 0));
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = kc;
        }
    }
    return best;
}

struct Plan {
    int kc, n_st, mu;
    int full_tiles, tail_k, tail_big;  // tail split (tail_k > 0), see GemmArgs
    bool split;        // some tile's K range is cut: counters and partials in use
    int64_t n_units;
    int64_t Mp;        // activation rows seen by the GEMM
    size_t ctr_off, ctr_bytes, part_off, gq_off, gs_off, gu_off, bytes;
};

int64_t uniform_cost(int64_t n_tiles, int64_t nsb, int kc, int sms) {
    const int64_t len = (nsb + kc - 1) / kc;
    return (n_tiles * kc + sms - 1) / sms * (100 * len + 235 + (kc > 1 ? 270 : 0));
}

// Tail split, in the cost units of choose_kc: every CTA runs full_tiles / SMs whole
// tiles, then one piece of a tail tile.  Applies when the tiles left after the whole
// rounds can each be cut into 2..15 pieces of at least 4 super-blocks that number
// exactly one per SM.  Returns the cost, or -1 when it does not apply.
int64_t tail_plan(int64_t n_tiles, int64_t nsb, int sms, int* full_tiles, int* tail_k, int* tail_big) {
    const int64_t rounds = n_tiles / sms, n_tail = n_tiles - rounds * sms;
    if (n_tail == 0) return -1;
    const int64_t k = sms / n_tail, big = sms - k * n_tail;
    if (k < 2 || k + (big > 0) > 15 || nsb / (k + (big > 0)) < 4) return -1;
    *full_tiles = (int)(rounds * sms);
    *tail_k = (int)k;
    *tail_big = (int)big;
    return rounds * (100 * nsb + 235) + 100 * ((nsb + k - 1) / k) + 235 + 270;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// The arrival counters are the only workspace contents that persist from one call to
// the next, so they sit in a fixed prefix that no call's partial sums or gathered rows
// ever overlap, whatever its shape: calls of different shapes can share a workspace.
constexpr size_t CTR_REGION = (size_t)64 << 10;

// K: the weight matrix's width in the kernel's form (2K for Q5_K); K_act: the
// activation width (the gathered requested rows are K_act wide).
Plan make_plan(int64_t n_tiles, int64_t K, int64_t M, int64_t n_rows, int sms, int64_t K_act) {
    Plan p;
    const int64_t nsb = K / QK, nsb_act = K_act / QK;
    p.Mp = round_up(n_rows > 0 ? n_rows : M, 16);
    p.kc = choose_kc(n_tiles, nsb, sms);
    p.full_tiles = p.tail_k = p.tail_big = 0;
    const int64_t tail_cost = tail_plan(n_tiles, nsb, sms, &p.full_tiles, &p.tail_k, &p.tail_big);
    const int64_t tail_units = (n_tiles / sms + 1) * sms * ((p.Mp + UNIT_TOKENS - 1) / UNIT_TOKENS);
    if (tail_cost < 0 || tail_cost >= uniform_cost(n_tiles, nsb, p.kc, sms) || tail_units >= (1LL << 31) ||
        nsb * 16 >= (1LL << 31))
        p.full_tiles = p.tail_k = p.tail_big = 0;
    if (p.tail_k > 0) p.kc = 1;
    p.split = p.kc > 1 || p.tail_k > 0;
    p.n_st = (int)((p.Mp + UNIT_TOKENS - 1) / UNIT_TOKENS);
    p.mu = (int)round_up((p.Mp + p.n_st - 1) / p.n_st, 16);
    p.n_units = p.tail_k > 0 ? (int64_t)(p.full_tiles + sms) * p.n_st : n_tiles * p.n_st * p.kc;
    size_t off = 0;
    p.ctr_off = off;
    p.ctr_bytes = (size_t)n_tiles * p.n_st * 4;  // one arrival counter per (tile, token super-tile)
    off += p.ctr_bytes > CTR_REGION ? align256(p.ctr_bytes) : CTR_REGION;
    p.part_off = off;
    if (p.kc > 1) off += align256((size_t)n_tiles * p.n_st * p.kc * p.mu * TROWS * 4);
    if (p.tail_k > 0) off += align256((size_t)sms * p.n_st * p.mu * TROWS * 4);
    p.gq_off = p.gs_off = p.gu_off = off;
    if (n_rows > 0) {
        p.gq_off = off;
        off += align256((size_t)p.Mp * K_act);
        p.gs_off = off;
        off += align256((size_t)nsb_act * p.Mp * 4);
        p.gu_off = off;
        off += align256((size_t)nsb_act * p.Mp * 64);
    }
    p.bytes = (p.split || n_rows > 0) ? off : 0;
    return p;
}

template <int QT, bool DBG, bool TAIL>
int run_gemm(GemmArgs& a, cudaStream_t s) {
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    constexpr size_t smem = gemm_smem_bytes<QT>();
    const int slot = (QT == 12 ? 0 : 4) + (DBG ? 2 : 0) + (TAIL ? 1 : 0);
    if (!g_attr_done[dev][slot]) {
        if (cudaFuncSetAttribute(qgemm_kernel<QT, DBG, TAIL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return DLLM_ERR_CUDA;
        // the warpgroups' setmaxnreg split must fit in the registers the CTA launches with
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, qgemm_kernel<QT, DBG, TAIL>) != cudaSuccess) return DLLM_ERR_CUDA;
        if (fa.numRegs * GEMM_THREADS < REG_SPLIT_TOTAL || fa.maxThreadsPerBlock < GEMM_THREADS)
            return DLLM_ERR_UNSUPPORTED;
        g_attr_done[dev][slot] = true;
    }
    const int64_t units = a.n_units;
    const int grid = (int)(units < g_num_sms[dev] ? units : g_num_sms[dev]);
    if (launch_pdl(qgemm_kernel<QT, DBG, TAIL>, dim3(grid), dim3(GEMM_THREADS), smem, s, a) != cudaSuccess) {
        (void)cudaGetLastError();
        return DLLM_ERR_CUDA;
    }
    return launch_status();
}

// Q5_K runs on the Q4_K kernel in its exact two-super-block form (see repack_q5k_kernel):
// weight width 2K, 2 x 144 repacked bytes per 256 weights.
int64_t kernel_k(dllm_qtype t, int64_t K) { return t == DLLM_Q5_K ? 2 * K : K; }
// Q8_0: the int8 codes (256 bytes) and eight f16 block scales per 256 weights of a row.
size_t repacked_per_sb(dllm_qtype t) {
    return t == DLLM_Q4_K ? Q4K_BLOCK : t == DLLM_Q5_K ? 2 * Q4K_BLOCK : t == DLLM_Q8_0 ? 272 : Q6K_BLOCK;
}

int check_shape(dllm_qtype t, int64_t N, int64_t K) {
    if (t != DLLM_Q4_K && t != DLLM_Q5_K && t != DLLM_Q6_K && t != DLLM_Q8_0) return DLLM_ERR_ARG;
    if (N <= 0 || K <= 0 || N % TROWS || K % QK) return DLLM_ERR_ARG;
    if (N / TROWS > (1LL << 30) || K / QK > (1 << 20)) return DLLM_ERR_ARG;
    return DLLM_OK;
}

int check_act(const int8_t* q, const float* scale, const uint8_t* sums, int64_t M) {
    if (!q || !scale || !sums || M <= 0) return DLLM_ERR_ARG;
    if (!aligned16(q) || !aligned16(scale) || !aligned16(sums)) return DLLM_ERR_ALIGN;
    return DLLM_OK;
}

// ---------------------------------------------------------------- Q8_0
bool g_q80_attr_done[MAX_DEV];

// Workspace of a Q8_0 GEMM: only the gathered requested rows (codes, scales, sums).
size_t q80_workspace(int64_t K, int64_t n_rows) {
    if (n_rows <= 0) return 0;
    const int64_t Mp = round_up(n_rows, 16), nsb = K / QK;
    return align256((size_t)Mp * K) + align256((size_t)nsb * Mp * 4) + align256((size_t)nsb * Mp * 64);
}

// The Q8_0 codes plane int8 [N][K] as a 2-D tensor with boxes of 128 bytes x 128 rows,
// 128-byte swizzled; the last few maps are kept per host thread.
bool q80_codes_map(CUtensorMap* m, const void* base, int64_t N, int64_t K) {
    struct Entry {
        const void* base;
        int64_t N, K;
        CUtensorMap map;
    };
    constexpr int NE = 8;
    thread_local Entry cache[NE] = {};
    thread_local int next = 0;
    for (int i = 0; i < NE; i++)
        if (cache[i].base == base && cache[i].N == N && cache[i].K == K) {
            *m = cache[i].map;
            return true;
        }
    const EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {128, (cuuint32_t)TROWS};
    const cuuint32_t estr[2] = {1, 1};
    if (fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    cache[next] = {base, N, K, *m};
    next = (next + 1) % NE;
    return true;
}

// One Q8_0 projection (rows: gathered into the workspace first, as for the K-quants).
// stall != 0 is the failure test: the producer issues no copy.
int q80_gemm(const void* w, int64_t N, int64_t K, const int8_t* q, const float* scale, const uint8_t* sums,
             int64_t M, const int32_t* rows, int64_t n_rows, float* out, int64_t ldo, void* workspace,
             size_t workspace_bytes, cudaStream_t s, int stall) {
    int rc = check_shape(DLLM_Q8_0, N, K);
    if (rc) return rc;
    if ((rc = check_act(q, scale, sums, M))) return rc;
    if (!w || !out || ldo < N) return DLLM_ERR_ARG;
    if (!aligned16(w) || !aligned16(out) || ldo % 4) return DLLM_ERR_ALIGN;
    if (rows && (n_rows < 1 || n_rows > 32)) return DLLM_ERR_ARG;
    if (rows && !aligned16(rows)) return DLLM_ERR_ALIGN;
    if (M > (1LL << 31)) return DLLM_ERR_ARG;
    if (workspace && !aligned16(workspace)) return DLLM_ERR_ALIGN;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t nsb = K / QK;
    const int64_t Mp = round_up(rows ? n_rows : M, 16);
    if (rows) {
        const size_t need = q80_workspace(K, n_rows);
        if (!workspace || workspace_bytes < need) return DLLM_ERR_WORKSPACE;
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        int8_t* gq = reinterpret_cast<int8_t*>(ws);
        float* gs = reinterpret_cast<float*>(ws + align256((size_t)Mp * K));
        uint8_t* gu = ws + align256((size_t)Mp * K) + align256((size_t)nsb * Mp * 4);
        if (launch_pdl(gather_rows_kernel, dim3(grid_for(nsb * Mp * 21, 256)), dim3(256), 0, s, q, scale, sums, M,
                       round_up(M, 16), rows, (int32_t)n_rows, Mp, (int32_t)nsb, gq, gs, gu) != cudaSuccess) {
            (void)cudaGetLastError();
            return DLLM_ERR_CUDA;
        }
        if ((rc = launch_status())) return rc;
        q = gq;
        scale = gs;
    }
    if (!g_q80_attr_done[dev]) {
        if (cudaFuncSetAttribute(q80_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Q80_SMEM) !=
            cudaSuccess)
            return DLLM_ERR_CUDA;
        g_q80_attr_done[dev] = true;
    }
    CUtensorMap tw;
    if (!q80_codes_map(&tw, w, N, K)) return DLLM_ERR_CUDA;
    Q80Args a;
    memset(&a, 0, sizeof(a));
    a.w = static_cast<const uint8_t*>(w);
    a.q = q;
    a.scale = scale;
    a.out = out;
    a.ldo = ldo;
    a.n_tiles = (int32_t)(N / TROWS);
    a.nsb = (int32_t)nsb;
    a.n_tok = (int32_t)((Mp + Q80_TOK - 1) / Q80_TOK);
    a.n_units = (int64_t)a.n_tiles * a.n_tok;
    a.Mp = (int32_t)Mp;
    a.m_out = (int32_t)(rows ? n_rows : M);
    a.stall = stall;
    const int grid = (int)(a.n_units < g_num_sms[dev] ? a.n_units : g_num_sms[dev]);
    if (launch_pdl(q80_gemm_kernel, dim3(stall ? 1 : grid), dim3(Q80_THREADS), Q80_SMEM, s, tw, a) != cudaSuccess) {
        (void)cudaGetLastError();
        return DLLM_ERR_CUDA;
    }
    return launch_status();
}

}  // namespace

extern "C" {

int dllm_repacked_bytes(dllm_qtype t, int64_t N, int64_t K, size_t* out_bytes) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if (!out_bytes) return DLLM_ERR_ARG;
    *out_bytes = (size_t)N * (size_t)(K / QK) * repacked_per_sb(t);
    return DLLM_OK;
}

static int repack(dllm_qtype t, const void* src, int64_t N, int64_t K, void* dst, dllm_stream_t stream) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if (!src || !dst) return DLLM_ERR_ARG;
    if (!aligned16(dst)) return DLLM_ERR_ALIGN;
    const size_t bytes = (size_t)N * (K / QK) * repacked_per_sb(t);
    const size_t src_bytes = (size_t)N * (K / QK) *
                             (t == DLLM_Q4_K ? Q4K_BLOCK : t == DLLM_Q5_K ? Q5K_BLOCK : t == DLLM_Q8_0 ? 272 : Q6K_BLOCK);
    const uint8_t* s8 = static_cast<const uint8_t*>(src);
    const uint8_t* d8 = static_cast<const uint8_t*>(dst);
    if (s8 < d8 + bytes && d8 < s8 + src_bytes) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t chunks = (int64_t)(bytes / 16);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (t == DLLM_Q4_K)
        repack_q4k_kernel<<<grid_for(chunks, 256), 256, 0, s>>>(s8, N, K / QK, static_cast<uint8_t*>(dst));
    else if (t == DLLM_Q5_K)
        repack_q5k_kernel<<<grid_for(chunks, 256), 256, 0, s>>>(s8, N, K / QK, static_cast<uint8_t*>(dst));
    else if (t == DLLM_Q8_0)
        repack_q80_kernel<<<grid_for(N * K / 16 + N * (K / QK), 256), 256, 0, s>>>(s8, N, K,
                                                                                  static_cast<uint8_t*>(dst));
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
int dllm_repack_q5k(const void* g, int64_t N, int64_t K, void* dst, dllm_stream_t s) {
    return repack(DLLM_Q5_K, g, N, K, dst, s);
}
int dllm_repack_q80(const void* g, int64_t N, int64_t K, void* dst, dllm_stream_t s) {
    return repack(DLLM_Q8_0, g, N, K, dst, s);
}

int dllm_act_bytes(int64_t M, int64_t K, size_t* q_bytes, size_t* scale_bytes, size_t* sums_bytes) {
    if (M <= 0 || K <= 0 || K % QK || !q_bytes || !scale_bytes || !sums_bytes) return DLLM_ERR_ARG;
    const int64_t Mp = round_up(M, 16);
    *q_bytes = (size_t)Mp * K;
    *scale_bytes = (size_t)Mp * (K / QK) * 4;
    *sums_bytes = (size_t)Mp * (K / QK) * 64;
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
    if (launch_pdl(quantize_act_kernel, grid, dim3(256), 0, reinterpret_cast<cudaStream_t>(stream), x, M, ldx, Mp, q,
                   scale, sums) != cudaSuccess) {
        (void)cudaGetLastError();
        return DLLM_ERR_CUDA;
    }
    return launch_status();
}

int dllm_rmsnorm_quantize(const float* x, int64_t M, int64_t K, int64_t ldx, const float* gamma, float eps,
                          const int32_t* rows, int64_t n_rows, int8_t* q, float* scale, uint8_t* sums,
                          dllm_stream_t stream) {
    if (!x || !gamma || M <= 0 || K <= 0 || K % QK || K > (int64_t)RMS_MAX_SB * QK || ldx < K) return DLLM_ERR_ARG;
    if (!(eps > 0.0f) || !(eps < INFINITY)) return DLLM_ERR_ARG;
    if (rows ? n_rows <= 0 : n_rows != 0) return DLLM_ERR_ARG;
    const int64_t M_out = rows ? n_rows : M;
    int rc = check_act(q, scale, sums, M_out);
    if (rc) return rc;
    if (!aligned16(x) || !aligned16(gamma) || ldx % 4 || (rows && !aligned16(rows))) return DLLM_ERR_ALIGN;
    if (M_out > (1LL << 31) - 16) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t Mp = round_up(M_out, 16);
    bool wide = false;
    const int warps = rms_warps(Mp, K, g_num_sms[dev], &wide);
    if (launch_pdl(wide ? rmsnorm_quantize_kernel<RMS_WIDE_SBR, RMS_WIDE_WARPS> : rmsnorm_quantize_kernel<1, RMS_MAX_WARPS>,
                   dim3((unsigned)Mp), dim3((unsigned)(warps * 32)), 0,
                   reinterpret_cast<cudaStream_t>(stream), x, M_out, K, ldx, gamma, eps, rows, M, Mp, q, scale,
                   sums) != cudaSuccess) {
        (void)cudaGetLastError();
        return DLLM_ERR_CUDA;
    }
    return launch_status();
}

int dllm_swiglu_quantize(const float* gate, const float* up, int64_t M, int64_t K, int64_t ld, int8_t* q, float* scale,
                         uint8_t* sums, dllm_stream_t stream) {
    if (!gate || !up || M <= 0 || K <= 0 || K % QK || ld < K) return DLLM_ERR_ARG;
    int rc = check_act(q, scale, sums, M);
    if (rc) return rc;
    if (!aligned16(gate) || !aligned16(up) || ld % 4) return DLLM_ERR_ALIGN;
    if (M > (1LL << 31) - 16 || K / QK > 65535LL * FUSE_WARPS) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t Mp = round_up(M, 16);
    const dim3 grid((unsigned)Mp, (unsigned)((K / QK + FUSE_WARPS - 1) / FUSE_WARPS));
    if (launch_pdl(swiglu_quantize_kernel, grid, dim3(FUSE_WARPS * 32), 0, reinterpret_cast<cudaStream_t>(stream),
                   gate, up, M, K, ld, Mp, q, scale, sums) != cudaSuccess) {
        (void)cudaGetLastError();
        return DLLM_ERR_CUDA;
    }
    return launch_status();
}

int dllm_qgemm_workspace_bytes(dllm_qtype t, int64_t N, int64_t K, int64_t M, int64_t n_rows, size_t* bytes) {
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if (M <= 0 || n_rows < 0 || n_rows > 32 || !bytes) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    *bytes = t == DLLM_Q8_0 ? q80_workspace(K, n_rows) : make_plan(N / TROWS, kernel_k(t, K), M, n_rows, g_num_sms[dev], K).bytes;
    return DLLM_OK;
}

// Validates the activation arguments and fills the parts of the launch that do not
// depend on the weights; gathers requested rows into the workspace first.
static int gemm_common(GemmArgs& a, dllm_qtype t, int64_t N_total, int64_t K, const int8_t* q, const float* scale,
                       const uint8_t* sums, int64_t M, const int32_t* rows, int64_t n_rows, void* workspace,
                       size_t workspace_bytes, bool dbg, cudaStream_t s) {
    int rc = check_shape(t, N_total, K);
    if (rc) return rc;
    if ((rc = check_act(q, scale, sums, M))) return rc;
    if (rows && (n_rows < 1 || n_rows > 32)) return DLLM_ERR_ARG;
    if (rows && !aligned16(rows)) return DLLM_ERR_ALIGN;
    if (M > (1LL << 31)) return DLLM_ERR_ARG;
    if (workspace && !aligned16(workspace)) return DLLM_ERR_ALIGN;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    if (dbg && (t == DLLM_Q5_K || t == DLLM_Q8_0)) return DLLM_ERR_ARG;  // the integer view covers Q4_K and Q6_K
    Plan p = make_plan(N_total / TROWS, kernel_k(t, K), M, rows ? n_rows : 0, g_num_sms[dev], K);
    if (dbg) {  // integers per super-block: no chunk partials to combine
        p.kc = 1;
        p.full_tiles = p.tail_k = p.tail_big = 0;
        p.split = false;
        p.n_units = (N_total / TROWS) * p.n_st;
        if (!rows) p.bytes = 0;
    }
    if (p.bytes > 0 && (!workspace || workspace_bytes < p.bytes)) return DLLM_ERR_WORKSPACE;
    memset(&a, 0, sizeof(a));
    const int64_t nsb = K / QK;  // activation super-blocks
    a.nsb = (int32_t)(kernel_k(t, K) / QK);
    a.nsb_act = (int32_t)nsb;
    a.kc = p.kc;
    a.full_tiles = p.full_tiles;
    a.tail_k = p.tail_k;
    a.tail_big = p.tail_big;
    a.n_units = p.n_units;
    a.n_st = p.n_st;
    a.mu = p.mu;
    a.Mp = p.Mp;
    a.m_out = rows ? n_rows : M;
    a.q = q;
    a.scale = scale;
    a.sums = sums;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (p.split) {
        a.counters = reinterpret_cast<uint32_t*>(ws + p.ctr_off);
        a.partials = reinterpret_cast<float*>(ws + p.part_off);
    }
    if (rows) {
        int8_t* gq = reinterpret_cast<int8_t*>(ws + p.gq_off);
        float* gs = reinterpret_cast<float*>(ws + p.gs_off);
        uint8_t* gu = ws + p.gu_off;
        const int64_t work = nsb * p.Mp * 21;
        if (launch_pdl(gather_rows_kernel, dim3(grid_for(work, 256)), dim3(256), 0, s, q, scale, sums, M,
                       round_up(M, 16), rows, (int32_t)n_rows, p.Mp, (int32_t)nsb, gq, gs, gu) != cudaSuccess) {
            (void)cudaGetLastError();
            return DLLM_ERR_CUDA;
        }
        if ((rc = launch_status())) return rc;
        a.q = gq;
        a.scale = gs;
        a.sums = gu;
    }
    return DLLM_OK;
}

static int dispatch(GemmArgs& a, dllm_qtype t, bool dbg, cudaStream_t s) {
    // the debug integers never split K (uniform plan, one chunk); Q5_K runs as Q4_K
    if (t == DLLM_Q4_K || t == DLLM_Q5_K) {
        if (dbg) return run_gemm<12, true, false>(a, s);
        return a.tail_k > 0 ? run_gemm<12, false, true>(a, s) : run_gemm<12, false, false>(a, s);
    }
    if (dbg) return run_gemm<14, true, false>(a, s);
    return a.tail_k > 0 ? run_gemm<14, false, true>(a, s) : run_gemm<14, false, false>(a, s);
}

int dllm_qgemm(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
               const uint8_t* sums, int64_t M, const int32_t* rows, int64_t n_rows, float* out, int64_t ldo,
               void* workspace, size_t workspace_bytes, dllm_stream_t stream) {
    if (!w || !out || ldo < N) return DLLM_ERR_ARG;
    if (!aligned16(w) || !aligned16(out) || ldo % 4) return DLLM_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (t == DLLM_Q8_0)
        return q80_gemm(w, N, K, q, scale, sums, M, rows, n_rows, out, ldo, workspace, workspace_bytes, s, 0);
    GemmArgs a;
    int rc = gemm_common(a, t, N, K, q, scale, sums, M, rows, n_rows, workspace, workspace_bytes, false, s);
    if (rc) return rc;
    a.seg[0] = Segment{static_cast<const uint8_t*>(w), out, ldo, 0};
    a.nseg = 1;
    a.n_tiles = (int32_t)(N / TROWS);
    return dispatch(a, t, false, s);
}

int dllm_qkv_qgemm(const void* wq, const void* wk, const void* wv, dllm_qtype t, int64_t Nq, int64_t Nkv, int64_t K,
                   const int8_t* q, const float* scale, const uint8_t* sums, int64_t M, float* oq, int64_t ldo_q,
                   float* ok, float* ov, int64_t ldo_kv, void* workspace, size_t workspace_bytes,
                   dllm_stream_t stream) {
    int rc = check_shape(t, Nq, K);
    if (rc) return rc;
    if ((rc = check_shape(t, Nkv, K))) return rc;
    if (!wq || !wk || !oq || !ok || (wv && !ov) || ldo_q < Nq || ldo_kv < Nkv) return DLLM_ERR_ARG;
    if (!aligned16(wq) || !aligned16(wk) || (wv && !aligned16(wv)) || !aligned16(oq) || !aligned16(ok) ||
        (wv && !aligned16(ov)) || ldo_q % 4 || ldo_kv % 4)
        return DLLM_ERR_ALIGN;
    const int64_t N_total = Nq + (wv ? 2 : 1) * Nkv;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (t == DLLM_Q8_0) {  // one launch per projection, all on the same quantized activation
        if ((rc = q80_gemm(wq, Nq, K, q, scale, sums, M, nullptr, 0, oq, ldo_q, workspace, workspace_bytes, s, 0)))
            return rc;
        if ((rc = q80_gemm(wk, Nkv, K, q, scale, sums, M, nullptr, 0, ok, ldo_kv, workspace, workspace_bytes, s, 0)))
            return rc;
        return wv ? q80_gemm(wv, Nkv, K, q, scale, sums, M, nullptr, 0, ov, ldo_kv, workspace, workspace_bytes, s, 0)
                  : DLLM_OK;
    }
    GemmArgs a;
    rc = gemm_common(a, t, N_total, K, q, scale, sums, M, nullptr, 0, workspace, workspace_bytes, false, s);
    if (rc) return rc;
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
    return dispatch(a, t, false, s);
}

// ---------------------------------------------------------------- no-workspace GEMM
}  // extern "C"

namespace {

// The fixed scratch of dllm_qgemm_noalloc, in the library's own device memory.  A
// zero-initialized __device__ array is reserved (and zeroed) by the CUDA runtime
// when this module's device code is loaded on a device, so the library never calls
// an allocator for it.
__device__ __align__(256) uint8_t g_noalloc_scratch[DLLM_NOALLOC_SCRATCH_BYTES];

uint8_t* g_noalloc_addr[MAX_DEV];  // device address of the array, per device, once known

bool att_attributes(int dev) {
    if (!g_att_attr_done[dev]) {
        if (cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ATT_SMEM) !=
                cudaSuccess ||
            cudaFuncSetAttribute(attention_pp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ATT_PP_SMEM) != cudaSuccess)
            return false;
        g_att_attr_done[dev] = true;
    }
    return true;
}

int noalloc_scratch(int dev, uint8_t** ptr) {
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DLLM_ERR_CUDA;
        g_noalloc_addr[dev] = static_cast<uint8_t*>(p);
    }
    *ptr = g_noalloc_addr[dev];
    return DLLM_OK;
}

}  // namespace

extern "C" {

int dllm_qgemm_noalloc(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
                       const uint8_t* sums, int64_t M, const int32_t* rows, int64_t n_rows, float* out,
                       int64_t ldo, dllm_stream_t stream) {
    // Every argument check dllm_qgemm makes, before anything is queued on the stream.
    if (!w || !out || ldo < N) return DLLM_ERR_ARG;
    if (!aligned16(w) || !aligned16(out) || ldo % 4) return DLLM_ERR_ALIGN;
    int rc = check_shape(t, N, K);
    if (rc) return rc;
    if ((rc = check_act(q, scale, sums, M))) return rc;
    if (rows && (n_rows < 1 || n_rows > 32)) return DLLM_ERR_ARG;
    if (rows && !aligned16(rows)) return DLLM_ERR_ALIGN;
    if (M > (1LL << 31)) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const Plan p = make_plan(N / TROWS, kernel_k(t, K), M, rows ? n_rows : 0, g_num_sms[dev], K);
    if (p.bytes > DLLM_NOALLOC_SCRATCH_BYTES) return DLLM_ERR_SCRATCH_LIMIT;
    uint8_t* scratch;
    if ((rc = noalloc_scratch(dev, &scratch))) return rc;
    if (p.split &&
        cudaMemsetAsync(scratch + p.ctr_off, 0, p.ctr_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DLLM_ERR_CUDA;
    return dllm_qgemm(w, t, N, K, q, scale, sums, M, rows, n_rows, out, ldo, scratch, DLLM_NOALLOC_SCRATCH_BYTES,
                      stream);
}

int dllm_attention(const void* q, const void* k, const void* v, int64_t Lq, int64_t Lk, int64_t H, int64_t Hkv,
                   int64_t dh, float* o, dllm_stream_t stream) {
    if (Lq < 0 || Lk < 0 || H <= 0 || Hkv <= 0 || H % Hkv || dh != ATT_DH) return DLLM_ERR_ARG;
    if (Lq == 0) return DLLM_OK;
    if (!q || !k || !v || !o || Lk == 0) return DLLM_ERR_ARG;
    if (Lq > (1LL << 30) || Lk > (1LL << 30) || H > 65535) return DLLM_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DLLM_ERR_ALIGN;
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    if (!att_attributes(dev)) return DLLM_ERR_CUDA;
    // the two-tile kernel reads K and V in blocks of 64 keys
    const bool pp = att_tiles_per_cta(Lq, H, g_num_sms[dev]) == 2;
    const int kv_rows = pp ? ATT_PP_BK : ATT_BK;
    CUtensorMap tq, tk, tv;
    if (!cached_head_rows(&tq, q, Lq, H, ATT_BQ) || !cached_head_rows(&tk, k, Lk, Hkv, kv_rows) ||
        !cached_head_rows(&tv, v, Lk, Hkv, kv_rows))
        return DLLM_ERR_CUDA;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (pp) {
        const dim3 grid((unsigned)((Lq + ATT_PP_BQ - 1) / ATT_PP_BQ), (unsigned)H);
        e = launch_pdl(attention_pp_kernel, grid, dim3(ATT_PP_THREADS), ATT_PP_SMEM, s, tq, tk, tv, o, (int)Lq,
                       (int)Lk, (int)H, (int)(H / Hkv), 0);
    } else {
        const dim3 grid((unsigned)((Lq + ATT_BQ - 1) / ATT_BQ), (unsigned)H);
        e = launch_pdl(attention_kernel, grid, dim3(ATT_THREADS), ATT_SMEM, s, tq, tk, tv, o, (int)Lq, (int)Lk,
                       (int)H, (int)(H / Hkv), 0);
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return DLLM_ERR_CUDA;
    }
    return launch_status();
}

int dllm_debug_attention_stall(int two_tiles, dllm_stream_t stream) {
    // One CTA of either attention kernel whose producers issue no copy.  The tensor maps
    // cover the library's own scratch array and are never read; nothing is stored.
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    uint8_t* base;
    if ((rc = noalloc_scratch(dev, &base))) return rc;
    if (!att_attributes(dev)) return DLLM_ERR_CUDA;
    const int Lq = two_tiles ? 2 * ATT_BQ : ATT_BQ, Lk = ATT_BK;
    CUtensorMap tq, tkv;
    if (!encode_head_rows(&tq, base, Lq, 1, ATT_BQ) ||
        !encode_head_rows(&tkv, base, Lk, 1, two_tiles ? ATT_PP_BK : ATT_BK))
        return DLLM_ERR_CUDA;
    float* o = reinterpret_cast<float*>(base + ((size_t)1 << 20));
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e =
        two_tiles ? launch_pdl(attention_pp_kernel, dim3(1, 1), dim3(ATT_PP_THREADS), ATT_PP_SMEM, s, tq, tkv, tkv, o,
                               Lq, Lk, 1, 1, 1)
                  : launch_pdl(attention_kernel, dim3(1, 1), dim3(ATT_THREADS), ATT_SMEM, s, tq, tkv, tkv, o, Lq, Lk,
                               1, 1, 1);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return DLLM_ERR_CUDA;
    }
    return launch_status();
}

int dllm_debug_attention_tiles(int64_t Lq, int64_t H, int sms) {
    if (Lq < 1 || H < 1 || sms < 1) return DLLM_ERR_ARG;
    return att_tiles_per_cta(Lq, H, sms);
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
        case DLLM_ERR_SCRATCH_LIMIT: return "call needs more scratch than the fixed no-allocation array holds";
        case DLLM_ERR_SCALE_RANGE: return "a Q5_K block scale d with |d| >= 4096: 16 d is not a finite f16";
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
// (a_tmem != 0) or shared memory.  `issuers` warps each issue `iters` MMAs (eight
// per loop trip, addresses precomputed) into their own n_acc accumulators.
__global__ void __launch_bounds__(128, 1) bench_mma_kernel(int n, int n_acc, int a_tmem, int iters, int issuers,
                                                           unsigned long long* ns_out) {
    extern __shared__ __align__(1024) uint8_t bsm[];
    __shared__ uint32_t tbase;
    __shared__ __align__(8) uint64_t bar[4];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < (256 * 32 + 128 * 32) / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(bsm)[i] = 0x01010101u;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; i++) mbar_init(&bar[i], 1);
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
    const uint64_t t0 = globaltimer_ns();
    if (lane == 0 && warp < issuers) {
        const uint32_t id = idesc_i8(128, n, 0, 1);
        const uint64_t bd = sdesc_kmajor_noswz(smem_u32(bsm), 128, 256);
        const uint64_t ad = sdesc_kmajor_noswz(smem_u32(bsm + 256 * 32), 128, 256);
        uint32_t dk[8], ak[8];
#pragma unroll
        for (int k = 0; k < 8; k++) {
            dk[k] = tm + (uint32_t)(warp * n * n_acc + (k % n_acc) * n);
            ak[k] = tm + 448 + 8 * k;
        }
        if (a_tmem) {
            for (int i = 0; i < iters; i += 8) {
#pragma unroll
                for (int k = 0; k < 8; k++) mma_i8_ts(dk[k], ak[k], bd, id, 1);
            }
        } else {
            for (int i = 0; i < iters; i += 8) {
#pragma unroll
                for (int k = 0; k < 8; k++) mma_i8_ss(dk[k], ad, bd, id, 1);
            }
        }
        tc_commit(&bar[warp]);
        uint64_t tw = globaltimer_ns();
        while (!mbar_try_wait(&bar[warp], 0)) {
            if (globaltimer_ns() - tw > WAIT_LIMIT_NS) { set_err(ERR_TIMEOUT); break; }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) ns_out[blockIdx.x] = globaltimer_ns() - t0;
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
    if (t == DLLM_Q5_K) return DLLM_ERR_ARG;
    if (!w || !q || !dots || M <= 0) return DLLM_ERR_ARG;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int64_t work = M * N * (K / QK);
    subblock_dots_kernel<<<grid_for(work, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(w), (int)t, N, (int)(K / QK), q, M, round_up(M, 16), dots);
    return launch_status();
}

int dllm_debug_sb_ints(const void* w, dllm_qtype t, int64_t N, int64_t K, const int8_t* q, const float* scale,
                       const uint8_t* sums, int64_t M, int32_t* S, dllm_stream_t stream) {
    if (!w || !S) return DLLM_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    GemmArgs a;
    int rc = gemm_common(a, t, N, K, q, scale, sums, M, nullptr, 0, nullptr, 0, true, s);
    if (rc) return rc;
    a.seg[0] = Segment{static_cast<const uint8_t*>(w), nullptr, N, 0};
    a.nseg = 1;
    a.n_tiles = (int32_t)(N / TROWS);
    a.dbg_S = S;
    a.dbg_N = N;
    return dispatch(a, t, true, s);
}

int dllm_debug_bounded_wait(dllm_stream_t stream) {
    // One CTA of the Q4_K GEMM kernel on a one-tile problem whose producer issues
    // nothing.  No pointer in the arguments is dereferenced: every other role's first
    // wait runs out instead.
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.nseg = 1;
    a.n_tiles = 1;
    a.nsb = 1;
    a.nsb_act = 1;
    a.kc = 1;
    a.n_units = 1;
    a.Mp = 16;
    a.m_out = 16;
    a.n_st = 1;
    a.mu = 16;
    a.stall = 1;
    return run_gemm<12, false, false>(a, reinterpret_cast<cudaStream_t>(stream));
}

int dllm_debug_plan(int64_t n_tiles, int64_t K, int64_t M, int64_t n_rows, int sms, int64_t* out) {
    if (n_tiles <= 0 || n_tiles > (1LL << 30) || K <= 0 || K % QK || K / QK > (1 << 20) || M <= 0 ||
        M > (1LL << 31) || n_rows < 0 || n_rows > 32 || sms <= 0 || sms > 4096 || !out)
        return DLLM_ERR_ARG;
    const Plan p = make_plan(n_tiles, K, M, n_rows, sms, K);
    out[0] = p.kc;
    out[1] = p.full_tiles;
    out[2] = p.tail_k;
    out[3] = p.tail_big;
    out[4] = p.n_units;
    out[5] = p.n_st;
    out[6] = p.mu;
    out[7] = (int64_t)p.bytes;
    return DLLM_OK;
}

int dllm_bench_mma_i8(int n, int n_acc, int a_from_tmem, int issuers, int iters, int ctas,
                      unsigned long long* ns_out, dllm_stream_t stream) {
    if (n < 16 || n > 256 || n % 16 || n_acc < 1 || n_acc > 8 || issuers < 1 || issuers > 4 ||
        n * n_acc * issuers > 448 || iters < 8 || iters % 8 || ctas < 1 || ctas > 4096 || !ns_out)
        return DLLM_ERR_ARG;
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    const int smem = 120 * 1024;  // also keeps one CTA per SM
    if (cudaFuncSetAttribute(bench_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return DLLM_ERR_CUDA;
    bench_mma_kernel<<<ctas, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(n, n_acc, a_from_tmem, iters,
                                                                                  issuers, ns_out);
    return launch_status();
}

}  // extern "C"
