// Bidirectional attention over the canvas on the sm_100a tensor cores (mojo-dllm
// heatdrop card, "Key highlights": f16 tensor-core attention; Architecture page, "A
// forward pass", step 2: every position attends to all L positions, no causal mask).
//
//   o[i][h][:] = sum_j softmax_j(q[i][h] . k[j][g] / sqrt(dh)) v[j][g],  g = h / (H / Hkv)
//
// One CTA per (query tile of 128 rows, head), 7 warps:
//   warp 5      TMA producer of Q (once) and of K key blocks of 128 (two slots)
//   warp 6      TMA producer of V key blocks (two slots); rows past Lk (and query
//               rows past Lq) arrive as zeros
//   warp 4      one thread issues the MMAs and allocates tensor memory:
//               S(kb) = Q K(kb)^T   tcgen05 kind::f16, f32 in tensor memory (two slots
//                                   of 128 lanes x 128 key columns)
//               O += P(kb) V(kb)    kind::f16, f32 in tensor memory (128 x dh)
//               S(kb + 1) is issued before P(kb) is waited for, so the tensor core
//               works on the next block while the softmax threads work on this one
//   warps 0-3   softmax, thread = query row = tensor-memory lane: block maximum,
//               running maximum m (base-2 exponents), P = 2^(S c - m) rounded to f16
//               into one of two shared-memory slots, running sum l; O is rescaled in
//               tensor memory only when m is raised.  At the end O / l is stored.
// Keys beyond Lk score -inf; query rows beyond Lq are not stored.
//
// Shared-memory tiles:
//   Q, K, V  two TMA boxes of 64 head-dim values x 128 rows (16 KB each, 128-byte
//            rows, 128-byte swizzle).  For Q and K (row = query or key, K = head dim)
//            this is the K-major swizzled layout: 1024 bytes between 8-row atoms, a
//            K step of 16 values = 32 bytes along the row, the second box at +16 KB
//            for head-dim 64..127.  For V (row = key, column = head dim) the same
//            bytes are the MN-major swizzled B operand of P V: 64 head-dim values per
//            atom row, the second box 16 KB further along N, 1024 bytes between groups
//            of 8 keys (2048 per K step of 16 keys).  So V needs no transpose.
//   P        no swizzle, element (r, c) at ((r/8)*16 + c/8)*128 + (r%8)*16 + (c%8)*2,
//            written by the softmax threads (a quarter warp stores 128 contiguous
//            bytes): K-major, 128 bytes between core matrices along K, 2048 between
//            8-row groups.
#pragma once
#include <cuda.h>

#include "layout.cuh"

namespace dllm {

constexpr int ATT_DH = 128;       // head dimension (LLaDA-8B: 4096 / 32, Dream-7B: 3584 / 28)
constexpr int ATT_BQ = 128;       // queries per CTA (tensor-memory lanes)
constexpr int ATT_BK = 128;       // keys per block
constexpr int ATT_THREADS = 224;  // warps 0-3 softmax and output, warp 4 MMA issue, 5 Q and K, 6 V
constexpr int ATT_TILE = 128 * ATT_DH * 2;  // one 128 x 128 f16 tile, 32 KB
constexpr uint32_t ATT_TM_COLS = 512;       // S blocks: columns 0..127 and 128..255, O: 256..383
constexpr uint32_t ATT_TM_O = 256;
constexpr size_t ATT_SMEM = 7 * (size_t)ATT_TILE + 256;  // Q, K x2, V x2, P x2, barriers
// log2(e) / sqrt(128): scores times this are base-2 exponents.
constexpr float ATT_C = 0.12751743082459868f;
// The running maximum is raised (and O, l rescaled) only when a block maximum exceeds
// it by more than this many binades; until then P <= 2^8, which f16 holds exactly
// as well as any other value in its normal range.
constexpr float ATT_RESCALE_LOG2 = 8.0f;
constexpr uint64_t ATT_WAIT_NS = 2000000000ull;

// Byte offset of element (r, c) of the P tile.
__device__ __forceinline__ uint32_t att_off(int r, int c) {
    return (uint32_t)(((r >> 3) * (ATT_DH / 8) + (c >> 3)) * 128 + (r & 7) * 16 + (c & 7) * 2);
}

__device__ __forceinline__ bool att_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > ATT_WAIT_NS) {
            set_err(ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Bounded wait that runs also after another wait gave up: used before the CTA exits,
// for copies and MMAs already in flight.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > ATT_WAIT_NS) {
            set_err(ERR_TIMEOUT);
            return;
        }
}

// Lanes 0 and 1 of a producer warp each bring one 16 KB box (64 head-dim values x 128
// rows of one head, rows r0..r0+127) of a [rows][heads][128] f16 tensor into a tile;
// lane 0 has armed `bar` for the whole 32 KB before.
__device__ __forceinline__ void att_tma_tile(uint8_t* tile, const CUtensorMap* tmap, int head, int r0, uint64_t* bar,
                                             int lane) {
    if (lane < 2) tma_load_3d(tile + lane * 16384, tmap, 64 * lane, head, r0, bar);
}

// 2^x on the special-function unit (PTX ex2.approx.ftz: relative error below 2^-22,
// 2^-inf = 0, results below the f32 normal range flush to 0).
__device__ __forceinline__ float att_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


// Descriptors of the tiles.
__device__ __forceinline__ uint64_t att_qk_desc(const uint8_t* t, int kk) {
    return sdesc_sw128(smem_u32(t + (kk >> 2) * 16384 + (kk & 3) * 32), 16, 1024);
}
__device__ __forceinline__ uint64_t att_v_desc(const uint8_t* t, int kk) {
    return sdesc_sw128(smem_u32(t + kk * 2048), 16384, 1024);
}
__device__ __forceinline__ uint64_t att_p_desc(const uint8_t* t, int kk) {
    return sdesc_kmajor_noswz(smem_u32(t + kk * 256), 128, 2048);
}

// Tensor maps over q: f16 [Lq][H][128], k, v: f16 [Lk][Hkv][128] as 3-D tensors
// (head dim, head, row) with boxes of 8 x 1 x 128; o: f32 [Lq][H][128]; group = H / Hkv.
// Grid (ceil(Lq / 128), H).  Requires Lk >= 1.
//
// Buffers with two slots (index b = kb & 1 for key block kb): K, V, S (tensor
// memory), P.  Barriers, each completing once per use of its slot:
//   k_full[b], v_full[b]   TMA transaction count of the 32 KB tile
//   k_empty[b]             commit after Q K^T(kb): the K slot may be refilled
//   s_full[b]              the same commit: S(kb) is ready
//   p_full[b]              softmax threads, after P(kb) is in shared memory
//   o_done[b], v_empty[b]  commit after P V(kb): O holds blocks 0..kb, and the P and
//                          V slots may be refilled
// A wait on "use u of slot b" takes parity (u >> 1) & 1; no barrier can run two uses
// ahead of its slowest waiter, because each next use needs that waiter's own progress.
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, float* __restrict__ o, int Lq, int Lk, int H,
                     int group) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* const sQ = smem;
    uint8_t* const sK = smem + ATT_TILE;      // two slots
    uint8_t* const sV = smem + 3 * ATT_TILE;  // two slots
    uint8_t* const sP = smem + 5 * ATT_TILE;  // two slots
    uint64_t* const bars = reinterpret_cast<uint64_t*>(smem + 7 * ATT_TILE);
    uint64_t* const q_full = bars;
    uint64_t* const k_full = bars + 1;
    uint64_t* const v_full = bars + 3;
    uint64_t* const k_empty = bars + 5;
    uint64_t* const v_empty = bars + 7;
    uint64_t* const s_full = bars + 9;
    uint64_t* const p_full = bars + 11;
    uint64_t* const o_done = bars + 13;
    uint64_t* const fin = bars + 15;
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * ATT_BQ, h = blockIdx.y, hk = h / group;
    const int nkb = (Lk + ATT_BK - 1) / ATT_BK;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int b = 0; b < 2; b++) {
            mbar_init(&k_full[b], 1);
            mbar_init(&v_full[b], 1);
            mbar_init(&k_empty[b], 1);
            mbar_init(&v_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], ATT_BQ);
            mbar_init(&o_done[b], 1);
        }
        mbar_init(fin, 1);
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_slot, ATT_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    pdl_wait();  // q, k, v may come from the previous kernel on the stream

    if (warp >= 5) {
        // ---------------------------------------------------------------- TMA producers
        const bool is_k = warp == 5;
        if (is_k) {
            if (lane == 0) mbar_arrive_expect_tx(q_full, ATT_TILE);
            __syncwarp();
            att_tma_tile(sQ, &tq, h, q0, q_full, lane);
        }
        uint64_t* const full = is_k ? k_full : v_full;
        uint64_t* const empty = is_k ? k_empty : v_empty;
        const CUtensorMap* const tmap = is_k ? &tk : &tv;
        uint8_t* const dst = is_k ? sK : sV;
        int issued = 0;
        for (int kb = 0; kb < nkb; kb++) {
            const int b = kb & 1;
            if (kb >= 2 && !__all_sync(~0u, att_wait(&empty[b], ((kb >> 1) - 1) & 1))) break;
            if (lane == 0) mbar_arrive_expect_tx(&full[b], ATT_TILE);
            __syncwarp();
            att_tma_tile(dst + b * ATT_TILE, tmap, hk, kb * ATT_BK, &full[b], lane);
            issued = kb + 1;
        }
        // No copy may still be landing in shared memory when the CTA exits, also when
        // a wait ran out: wait for the last use of each slot (and for Q).
        if (lane == 0) {
            for (int kb = issued > 2 ? issued - 2 : 0; kb < issued; kb++) drain_wait(&full[kb & 1], (kb >> 1) & 1);
            if (is_k) drain_wait(q_full, 0);
        }
        __syncwarp();
    } else if (warp == 4) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_f16(ATT_BQ, ATT_BK);
            constexpr uint32_t ID_O = idesc_f16(ATT_BQ, ATT_DH) | (1u << 16);  // B (V) MN-major
            // S[b] = Q K^T for key block kb: 8 steps of K = 16 along the head dimension.
            auto issue_s = [&](int kb) -> bool {
                const int b = kb & 1;
                if (!att_wait(&k_full[b], (kb >> 1) & 1)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < ATT_DH / 16; kk++)
                    mma_f16_ss(tm + b * ATT_BK, att_qk_desc(sQ, kk), att_qk_desc(sK + b * ATT_TILE, kk), ID_S,
                               kk > 0);
                tc_commit(&s_full[b]);
                tc_commit(&k_empty[b]);
                return true;
            };
            bool ok = att_wait(q_full, 0) && issue_s(0);
            for (int kb = 0; ok && kb < nkb; kb++) {
                // S for the next block runs while the softmax threads work on this one.
                if (kb + 1 < nkb && !issue_s(kb + 1)) break;
                const int b = kb & 1;
                if (!att_wait(&p_full[b], (kb >> 1) & 1) || !att_wait(&v_full[b], (kb >> 1) & 1)) break;
                tc_fence_after();
                // O += P V: 8 steps of K = 16 keys.
#pragma unroll
                for (int kk = 0; kk < ATT_BK / 16; kk++)
                    mma_f16_ss(tm + ATT_TM_O, att_p_desc(sP + b * ATT_TILE, kk), att_v_desc(sV + b * ATT_TILE, kk),
                               ID_O, (kb | kk) != 0);
                tc_commit(&o_done[b]);
                tc_commit(&v_empty[b]);
            }
            // Every MMA issued above completes before the tensor memory is released,
            // also when a wait ran out.
            tc_commit(fin);
            drain_wait(fin, 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax, output
        const int row = threadIdx.x;  // query q0 + row, tensor-memory lane row
        const uint32_t tl = tm + ((uint32_t)(warp * 32) << 16);
        float m = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int kb = 0; kb < nkb; kb++) {
            const int b = kb & 1;
            ok = __all_sync(~0u, att_wait(&s_full[b], (kb >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[ATT_BK];
#pragma unroll
            for (int j = 0; j < ATT_BK / 16; j++) tmem_ld16(tl + b * ATT_BK + 16 * j, sr + 16 * j);
            tmem_wait_ld();
            // block maximum over the valid keys (eight independent chains)
            const int kvalid = Lk - kb * ATT_BK;  // >= 1
            float mx[8];
#pragma unroll
            for (int e = 0; e < 8; e++) mx[e] = -INFINITY;
#pragma unroll
            for (int j = 0; j < ATT_BK; j++) {
                const float x = j < kvalid ? __uint_as_float(sr[j]) : -INFINITY;
                sr[j] = __float_as_uint(x);
                mx[j & 7] = fmaxf(mx[j & 7], x);
            }
            const float bm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            const float mc = bm * ATT_C;
            const bool raise = kb == 0 || mc > m + ATT_RESCALE_LOG2;
            const float m_new = raise ? mc : m;
            // P(kb) = 2^(s c - m_new) in f16 pairs; l sums the unrounded weights.
            uint32_t pk[ATT_BK / 2];
            float ps[8];
#pragma unroll
            for (int e = 0; e < 8; e++) ps[e] = 0.0f;
#pragma unroll
            for (int j = 0; j < ATT_BK; j += 2) {
                const float p0 = att_ex2(fmaf(__uint_as_float(sr[j]), ATT_C, -m_new));
                const float p1 = att_ex2(fmaf(__uint_as_float(sr[j + 1]), ATT_C, -m_new));
                ps[(j >> 1) & 7] += p0 + p1;
                const __half2 hp = __floats2half2_rn(p0, p1);
                pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&hp);
            }
            const float ls = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            if (kb >= 2) {
                // P V(kb - 2) has read this P slot
                ok = __all_sync(~0u, att_wait(&o_done[b], ((kb - 2) >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
            }
            if (kb >= 1 && __any_sync(~0u, raise)) {
                // O must hold blocks 0..kb-1 before it is rescaled to the new maximum
                ok = __all_sync(~0u, att_wait(&o_done[b ^ 1], ((kb - 1) >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
                const float alpha = raise ? att_ex2(m - m_new) : 1.0f;
                l *= alpha;
#pragma unroll 1
                for (int j = 0; j < ATT_DH / 16; j++) {
                    uint32_t t[16];
                    tmem_ld16(tl + ATT_TM_O + 16 * j, t);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e++) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
                    tmem_st16(tl + ATT_TM_O + 16 * j, t);
                }
                tmem_wait_st();
            }
            l += ls;
            m = m_new;
            uint8_t* const pt = sP + b * ATT_TILE;
#pragma unroll
            for (int c8 = 0; c8 < ATT_BK / 8; c8++)
                *reinterpret_cast<uint4*>(pt + att_off(row, 8 * c8)) =
                    make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&p_full[b]);
        }
        if (ok) ok = __all_sync(~0u, att_wait(&o_done[(nkb - 1) & 1], ((nkb - 1) >> 1) & 1));
        if (ok) {
            tc_fence_after();
            const int qi = q0 + row;
            const float inv = 1.0f / l;
            float* dst = o + ((int64_t)qi * H + h) * ATT_DH;
#pragma unroll 1
            for (int j = 0; j < ATT_DH / 16; j++) {
                uint32_t t[16];
                tmem_ld16(tl + ATT_TM_O + 16 * j, t);
                tmem_wait_ld();
                if (qi < Lq) {
#pragma unroll
                    for (int e = 0; e < 4; e++)
                        reinterpret_cast<float4*>(dst + 16 * j)[e] =
                            make_float4(__uint_as_float(t[4 * e]) * inv, __uint_as_float(t[4 * e + 1]) * inv,
                                        __uint_as_float(t[4 * e + 2]) * inv, __uint_as_float(t[4 * e + 3]) * inv);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tm, ATT_TM_COLS);
    }
}

}  // namespace dllm
