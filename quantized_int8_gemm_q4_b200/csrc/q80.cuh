// Q8_0 x int8 projection GEMM on the sm_100a tensor cores.
//
// GGUF Q8_0 (mojo-dllm Architecture page, "Source map", quant/kquants.mojo row lists
// the formats): blocks of 32 weights with one f16 scale each, w = d_b * q, q int8.  With
// the int8 activation of one f32 scale per 256 elements:
//   out[m][n] = sum_sb da[m][sb] * sum_{b in sb} d[n][b] * dot_b[n][m]
//   dot_b     = sum_{k in block b} q[n][k] * qa[m][k]      (int32, exact)
// A 32-wide block is exactly one K step of an int8 MMA, and every block has its own
// scale, so each block's dot product goes to an accumulator of its own: per super-block
// eight accumulators of (128 weight rows x 32 tokens) in tensor memory, two sets of
// them so the MMAs of the next super-block run while the epilogue reads this one.  The
// accumulators are preset to the bits of 1.5 * 2^23 and the MMAs add to them, so each
// holds the f32 1.5 * 2^23 + dot exactly (|dot| <= 32 * 128 * 127 < 2^22); the epilogue
// subtracts 1.5 * 2^23 (exact), writes the preset back, and accumulates
// da * sum_b d_b * dot_b in f32 registers with packed two-token operations.
//
// The period of a super-block is set by the tensor pipe and by tensor-memory latency,
// not by HBM: an int8 MMA with A in shared memory takes ~110 cycles at N <= 128 whatever
// the thread that issues it (two issuing threads give no more), so the eight MMAs of a
// super-block take ~870 cycles; and each load -> wait -> preset -> wait round trip of
// tensor memory takes ~150-350 cycles with 16 warps, against ~425 B per cycle per SM of
// tensor-memory bandwidth that the epilogue uses only a third of.  Measured and kept
// out: 64-token units (one accumulator set with a release per quarter, N = 64 halving
// the MMAs per token) were slower because the epilogue round trips then sit on the
// path of every quarter, and one round trip for all eight blocks leaves the epilogue's
// arithmetic after the release, where it becomes the period.
//
// Repacked weights (dllm_repack_q80, same 272 bytes per 256 weights as GGUF):
//   codes  int8 [N][K] row-major, read by TMA in boxes of 128 bytes x 128 rows with the
//          128-byte swizzle (the K-major swizzled A operand: 1024 bytes between 8-row
//          groups, a K step of 32 codes = 32 bytes along the row, the super-block's
//          second 128 codes in a second box 16 KB further)
//   scales f16 [N/128][K/256][128 rows][8 blocks] after the codes (2 KB per tile
//          super-block, one bulk copy)
//
// One CTA per SM, persistent over work units (128 weight rows, 32 tokens, all of K);
// the units of one weight tile are consecutive, so the tile streams from HBM once and
// from L2 for the other token groups.  18 warps:
//   warp 0      producer: per super-block one stage of 5 (codes by TMA, scales, the
//               activation codes and scales by bulk copies), after the dependency wait
//   warp 1      one thread issues the 8 MMAs of a super-block (kind::i8, A and B from
//               shared memory, accumulating onto the preset), and the warp owns tensor
//               memory
//   warps 2-17  epilogue: the warp's tensor-memory lane quadrant is warp % 4 and its 8
//               tokens (warp - 2) / 4; it takes all eight blocks of its rows and tokens,
//               two blocks per tensor-memory round trip, so each output has one owner
//               and is stored straight from registers
#pragma once
#include <cuda.h>

#include "qgemm.cuh"

namespace dllm {

constexpr int Q80_TOK = 32;                    // tokens per unit (the MMA's N)
constexpr int Q80_STAGES = 5;
constexpr int Q80_SQ = TROWS * QK;             // codes of a tile super-block, 32 KB
constexpr int Q80_SA = Q80_TOK * QK;           // activation codes, 8 KB
constexpr int Q80_SD = TROWS * 8 * 2;          // block scales, 2 KB
constexpr int Q80_SS = Q80_TOK * 4;            // activation scales
constexpr int Q80_OFF_A = Q80_SQ;
constexpr int Q80_OFF_D = Q80_SQ + Q80_SA;
constexpr int Q80_OFF_S = Q80_OFF_D + Q80_SD;
constexpr int Q80_STAGE = (Q80_OFF_S + Q80_SS + 1023) / 1024 * 1024;
constexpr int Q80_EPI_WARP0 = 2;
constexpr int Q80_EPI_WARPS = 16;
constexpr int Q80_THREADS = 32 * (Q80_EPI_WARP0 + Q80_EPI_WARPS);
constexpr size_t Q80_SMEM = (size_t)Q80_STAGES * Q80_STAGE + 256;
constexpr uint64_t Q80_WAIT_NS = 2000000000ull;

struct Q80Args {
    const uint8_t* w;   // repacked weights (codes, then scales)
    const int8_t* q;    // activation codes, tiled like quantize_act's output
    const float* scale; // activation scales [K/256][Mp]
    float* out;         // [m_out][ldo]
    int64_t ldo;
    int64_t n_units;
    int32_t n_tiles, nsb, n_tok;  // weight tiles, super-blocks, token groups of 32
    int32_t Mp, m_out;
    int32_t stall;                // failure test only: the producer issues nothing
};

// Bounded wait; the first poll does not read the timer.
__device__ __forceinline__ bool q80_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > Q80_WAIT_NS) {
            set_err(ERR_TIMEOUT);
            return false;
        }
    return true;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Unit u: weight tile u / n_tok, tokens 32 (u % n_tok) .. + 32 (16 in a last group of 16).
__device__ __forceinline__ void q80_unit(const Q80Args& a, int64_t u, int& tile, int& m0, int& ntok) {
    tile = (int)(u / a.n_tok);
    m0 = (int)(u % a.n_tok) * Q80_TOK;
    ntok = min(Q80_TOK, a.Mp - m0);
}

// 32 lanes x 8 consecutive 32-bit columns, all set to v.
__device__ __forceinline__ void tmem_st8_same(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr), "r"(v)
                 : "memory");
}

// Barriers (stage st = g % Q80_STAGES, accumulator set c = g & 1 for the CTA's g-th
// super-block):
//   full[st]     transaction bytes of the stage's copies
//   empty[st]    the issuer's commit (MMAs read the codes) and the 16 epilogue warps (they
//                read the scales)
//   acc_full[c]  the issuer's commit after the 8 MMAs
//   acc_empty[c] the 16 epilogue warps, once their columns are in registers and preset
//                again (use 0: the first preset, before any MMA)
//   fin          the issuer's last commit, before tensor memory is freed
// Each waits with parity (use & 1) where use counts the barrier's completions; no
// barrier runs two uses ahead of a waiter, because its next use needs that waiter.
__global__ void __launch_bounds__(Q80_THREADS, 1) q80_gemm_kernel(const __grid_constant__ CUtensorMap tw,
                                                                 const __grid_constant__ Q80Args a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* const bars = reinterpret_cast<uint64_t*>(smem + Q80_STAGES * Q80_STAGE);
    uint64_t* const full = bars;                      // [Q80_STAGES]
    uint64_t* const empty = bars + Q80_STAGES;        // [Q80_STAGES]
    uint64_t* const acc_full = bars + 2 * Q80_STAGES; // [2]
    uint64_t* const acc_empty = acc_full + 2;         // [2]
    uint64_t* const fin = acc_full + 4;
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 5);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < Q80_STAGES; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1 + Q80_EPI_WARPS);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], Q80_EPI_WARPS);
        }
        mbar_init(fin, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    if (threadIdx.x == 0) pdl_trigger();
    const uint8_t* const dplane = a.w + (size_t)a.n_tiles * TROWS * a.nsb * QK;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            pdl_wait();  // activations (and the output) may belong to the previous kernel
            uint32_t g = 0, issued = 0;
            bool ok = true;
            const int64_t n_prod = a.stall ? 0 : a.n_units;
            for (int64_t u = blockIdx.x; ok && u < n_prod; u += gridDim.x) {
                int tile, m0, ntok;
                q80_unit(a, u, tile, m0, ntok);
                for (int s = 0; s < a.nsb; s++, g++) {
                    const int st = (int)(g % Q80_STAGES);
                    if (g >= Q80_STAGES && !q80_wait(&empty[st], ((g / Q80_STAGES) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t* const sb = smem + st * Q80_STAGE;
                    mbar_arrive_expect_tx(&full[st], Q80_SQ + ntok * QK + Q80_SD + ntok * 4);
                    tma_load_2d(sb, &tw, s * QK, tile * TROWS, &full[st]);
                    tma_load_2d(sb + Q80_SQ / 2, &tw, s * QK + 128, tile * TROWS, &full[st]);
                    bulk_g2s(sb + Q80_OFF_A, a.q + ((size_t)s * a.Mp + m0) * QK, ntok * QK, &full[st]);
                    bulk_g2s(sb + Q80_OFF_D, dplane + ((size_t)tile * a.nsb + s) * Q80_SD, Q80_SD, &full[st]);
                    bulk_g2s(sb + Q80_OFF_S, a.scale + (size_t)s * a.Mp + m0, ntok * 4, &full[st]);
                    issued = g + 1;
                }
            }
            // no copy may still be landing when the CTA exits: wait for the last stages
            for (uint32_t h = issued > Q80_STAGES ? issued - Q80_STAGES : 0; h < issued; h++)
                (void)q80_wait(&full[h % Q80_STAGES], (h / Q80_STAGES) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; ok && u < a.n_units; u += gridDim.x) {
                int tile, m0, ntok;
                q80_unit(a, u, tile, m0, ntok);
                const uint32_t id = idesc_i8(TROWS, ntok, 1, 1);
                for (int s = 0; s < a.nsb; s++, g++) {
                    const int st = (int)(g % Q80_STAGES), c = (int)(g & 1);
                    if (!q80_wait(&full[st], (g / Q80_STAGES) & 1) || !q80_wait(&acc_empty[c], (g >> 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* const sb = smem + st * Q80_STAGE;
                    const uint64_t da = sdesc_sw128(smem_u32(sb), 16, 1024);
                    const uint64_t db = sdesc_kmajor_noswz(smem_u32(sb + Q80_OFF_A), 128, 2048);
#pragma unroll
                    for (int b = 0; b < 8; b++)
                        mma_i8_ss(tm + 256 * c + 32 * b, da + (uint64_t)((b >> 2) * 1024 + (b & 3) * 2),
                                  db + (uint64_t)(16 * b), id, 1u);
                    tc_commit(&acc_full[c]);
                    tc_commit(&empty[st]);
                }
            }
            tc_commit(fin);
            (void)q80_wait(fin, 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        // warp: lane quadrant warp % 4 (rows 32 qd + lane), tokens 8 tg .. 8 tg + 7 of the
        // unit, all eight blocks of every super-block
        pdl_wait();  // the output may still be in use by the previous kernel
        const int qd = warp & 3, tg = (warp - Q80_EPI_WARP0) >> 2;
        const int row = 32 * qd + lane;
        const uint32_t tcol = tm + ((uint32_t)(32 * qd) << 16) + 8 * tg;  // + 256 c + 32 b
        // first preset of this warp's columns in both accumulator sets
#pragma unroll
        for (int cb = 0; cb < 16; cb++) tmem_st8_same(tcol + 32 * cb, MAGIC_BITS);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&acc_empty[0]);
            mbar_arrive(&acc_empty[1]);
        }
        const float2 nM = make_float2(-MAGIC, -MAGIC);
        uint32_t g = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; ok && u < a.n_units; u += gridDim.x) {
            int tile, m0, ntok;
            q80_unit(a, u, tile, m0, ntok);
            // warp-uniform: a last group of 16 tokens leaves token groups 2 and 3 idle (the
            // MMAs of N = 16 never write their columns, which keep the preset)
            const bool act = 8 * tg < ntok;
            float2 acc[4];
#pragma unroll
            for (int j = 0; j < 4; j++) acc[j] = make_float2(0.0f, 0.0f);
            for (int s = 0; s < a.nsb; s++, g++) {
                const int st = (int)(g % Q80_STAGES), c = (int)(g & 1);
                ok = __all_sync(~0u, q80_wait(&acc_full[c], (g >> 1) & 1) &&
                                         q80_wait(&full[st], (g / Q80_STAGES) & 1));
                if (!ok) break;
                tc_fence_after();
                const uint8_t* const sb = smem + st * Q80_STAGE;
                const uint4 dw = *reinterpret_cast<const uint4*>(sb + Q80_OFF_D + row * 16);
                const uint32_t dh[4] = {dw.x, dw.y, dw.z, dw.w};
                // two blocks at a time: into registers, preset again, folded into the
                // weighted sums t, the next two blocks' load issued before this pair's
                // arithmetic; the accumulators are free for the MMAs of super-block g + 2
                // once the last two blocks are preset
                float2 t[4];
                uint32_t x[2][2][8];
                if (act) {
                    tmem_ld8(tcol + 256 * c, x[0][0]);
                    tmem_ld8(tcol + 256 * c + 32, x[0][1]);
                }
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    if (act) {
                        tmem_wait_ld();
#pragma unroll
                        for (int b = 0; b < 2; b++) tmem_st8_same(tcol + 256 * c + 32 * (2 * h + b), MAGIC_BITS);
                        if (h < 3) {
#pragma unroll
                            for (int b = 0; b < 2; b++)
                                tmem_ld8(tcol + 256 * c + 32 * (2 * h + 2 + b), x[(h + 1) & 1][b]);
                        }
                    }
                    if (h == 3) {
                        if (act) tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&acc_empty[c]);
                    }
                    if (act) {
#pragma unroll
                        for (int b = 0; b < 2; b++) {
                            const float2 d2 = __half22float2(*reinterpret_cast<const __half2*>(&dh[h]));
                            const float d = (b & 1) ? d2.y : d2.x;
                            const float2 dd = make_float2(d, d);
#pragma unroll
                            for (int i = 0; i < 4; i++) {
                                const float2 X = __fadd2_rn(make_float2(__uint_as_float(x[h & 1][b][2 * i]),
                                                                        __uint_as_float(x[h & 1][b][2 * i + 1])),
                                                            nM);
                                t[i] = (h == 0 && b == 0) ? __fmul2_rn(dd, X) : __ffma2_rn(dd, X, t[i]);
                            }
                        }
                    }
                }
                const float4 s0 = *reinterpret_cast<const float4*>(sb + Q80_OFF_S + 32 * tg);
                const float4 s1 = *reinterpret_cast<const float4*>(sb + Q80_OFF_S + 32 * tg + 16);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                if (act) {
                    acc[0] = __ffma2_rn(make_float2(s0.x, s0.y), t[0], acc[0]);
                    acc[1] = __ffma2_rn(make_float2(s0.z, s0.w), t[1], acc[1]);
                    acc[2] = __ffma2_rn(make_float2(s1.x, s1.y), t[2], acc[2]);
                    acc[3] = __ffma2_rn(make_float2(s1.z, s1.w), t[3], acc[3]);
                }
            }
            if (ok && act) {
                const int cnt = min(ntok, a.m_out - m0) - 8 * tg;
                float* const dst = a.out + (int64_t)(m0 + 8 * tg) * a.ldo + (int64_t)tile * TROWS + row;
#pragma unroll
                for (int j = 0; j < 8; j++)
                    if (j < cnt) dst[(int64_t)j * a.ldo] = (j & 1) ? acc[j >> 1].y : acc[j >> 1].x;
            }
        }
        tmem_wait_st();  // a wait that ran out may leave presets in flight
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

// GGUF Q8_0 rows ([N][K/32] blocks of 34 bytes: d f16, 32 int8) -> the codes plane
// [N][K] and the scales plane [N/128][K/256][128][8] f16.  One thread per 16 output
// bytes of the codes plane, or per row super-block of the scales plane.
__global__ void repack_q80_kernel(const uint8_t* __restrict__ src, int64_t N, int64_t K, uint8_t* __restrict__ dst) {
    const int64_t nb = K / 32;
    const int64_t code_chunks = N * K / 16, scale_items = N * (K / QK);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < code_chunks + scale_items;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < code_chunks) {
            const int64_t n = i / (K / 16), k0 = (i % (K / 16)) * 16;
            const uint8_t* blk = src + (n * nb + k0 / 32) * 34 + 2 + (k0 % 32);
            alignas(16) uint8_t v[16];
#pragma unroll
            for (int j = 0; j < 16; j++) v[j] = blk[j];
            *reinterpret_cast<uint4*>(dst + n * K + k0) = *reinterpret_cast<const uint4*>(v);
        } else {
            const int64_t r = i - code_chunks;  // (row n, super-block s)
            const int64_t n = r / (K / QK), s = r % (K / QK);
            alignas(16) uint16_t d[8];
#pragma unroll
            for (int b = 0; b < 8; b++) {
                const uint8_t* blk = src + (n * nb + s * 8 + b) * 34;
                d[b] = (uint16_t)(blk[0] | (blk[1] << 8));
            }
            uint8_t* o = dst + N * K + (((n / TROWS) * (K / QK) + s) * TROWS + (n % TROWS)) * 16;
            *reinterpret_cast<uint4*>(o) = *reinterpret_cast<const uint4*>(d);
        }
    }
}

}  // namespace dllm
