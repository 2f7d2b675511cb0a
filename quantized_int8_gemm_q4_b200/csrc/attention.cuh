// Bidirectional attention over the canvas on the sm_100a tensor cores (mojo-dllm
// heatdrop card, "Key highlights": f16 tensor-core attention; Architecture page, "A
// forward pass", step 2: every position attends to all L positions, no causal mask).
//
//   o[i][h][:] = sum_j softmax_j(q[i][h] . k[j][g] / sqrt(dh)) v[j][g],  g = h / (H / Hkv)
//
// One CTA per (query tile of 128 rows, head), 12 warps:
//   warp 9      TMA producer of Q (once) and of K key blocks of 128 (two slots)
//   warp 10     TMA producer of V key blocks (two slots); rows past Lk (and query
//               rows past Lq) arrive as zeros
//   warp 8      one thread issues S(kb) = Q K(kb)^T (tcgen05 kind::f16, f32 in tensor
//               memory, two slots of 128 lanes x 128 key columns), as soon as K(kb) is
//               in and the softmax of block kb - 2 has left the slot; the warp
//               allocates tensor memory.  So the tensor core computes the next block's
//               scores while the softmax threads work on this one.
//   warp 11     one thread issues O += P(kb) V(kb) (kind::f16 with P read from tensor
//               memory, f32 in tensor memory, 128 x dh).  Two issuing threads,
//               because one thread issues a 128 x 128 x 16 MMA no faster than the
//               tensor core runs it.
//   warps 0-7   softmax, query row = tensor-memory lane 32 (w % 4) + lane; warps w and
//               w + 4 take key columns (and head-dim columns of O) 0..63 and 64..127
//               of the same rows and swap their half-block maxima through shared
//               memory and a named barrier of the two warps: running maximum m (base-2
//               exponents), P = 2^(S c - m) rounded to f16 into one of two
//               tensor-memory slots, running half sums of P; O is rescaled in tensor
//               memory only when m is raised.  At the end the two halves of l are
//               added and O / l is stored.
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
// P lives in tensor memory, one row per lane, two f16 keys per 32-bit column: the A
// operand of P V read from tensor memory (8 columns per K step of 16 keys).
#pragma once
#include <cuda.h>

#include "layout.cuh"

namespace dllm {

constexpr int ATT_DH = 128;       // head dimension (LLaDA-8B: 4096 / 32, Dream-7B: 3584 / 28)
constexpr int ATT_BQ = 128;       // queries per CTA (tensor-memory lanes)
constexpr int ATT_BK = 128;       // keys per block
constexpr int ATT_SOFTMAX_WARPS = 8;            // two per query-row quadrant, one per half of the columns
constexpr int ATT_MMA_WARP = ATT_SOFTMAX_WARPS;  // one thread issues Q K^T; the warp owns tensor memory
constexpr int ATT_K_WARP = ATT_MMA_WARP + 1;     // TMA producer of Q and K
constexpr int ATT_V_WARP = ATT_MMA_WARP + 2;     // TMA producer of V
constexpr int ATT_PV_WARP = ATT_MMA_WARP + 3;    // one thread issues P V
constexpr int ATT_THREADS = 32 * (ATT_SOFTMAX_WARPS + 4);
constexpr int ATT_TILE = 128 * ATT_DH * 2;  // one 128 x 128 f16 tile, 32 KB
// Tensor memory: S slots at columns 0..127 and 128..255 (f32), O at 256..383 (f32), P
// slots at 384..447 and 448..511 (f16 pairs, 128 keys per row).
constexpr uint32_t ATT_TM_COLS = 512;
constexpr uint32_t ATT_TM_O = 256;
constexpr uint32_t ATT_TM_P = 384;
// Q, K x2, V x2, barriers and tensor-memory address, exchange values [2][2][128]
constexpr size_t ATT_SMEM = 5 * (size_t)ATT_TILE + 256 + 4 * 128 * 4;
// log2(e) / sqrt(128): scores times this are base-2 exponents.
constexpr float ATT_C = 0.12751743082459868f;
// The running maximum is raised (and O, l rescaled) only when a block maximum exceeds
// it by more than this many binades; until then P <= 2^8, which f16 holds exactly
// as well as any other value in its normal range.
constexpr float ATT_RESCALE_LOG2 = 8.0f;
constexpr uint64_t ATT_WAIT_NS = 2000000000ull;

// Bounded wait on a phase; the first poll does not read the timer (most waits in the
// pipeline find the phase already complete).
__device__ __forceinline__ bool att_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
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

// max(a, b, c) in one instruction (PTX max.f32 with three sources; -inf is the identity).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x on the special-function unit (PTX ex2.approx.ftz: relative error below 2^-22,
// 2^-inf = 0, results below the f32 normal range flush to 0).
__device__ __forceinline__ float att_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


// Descriptors of the tiles at their first K step; a K step adds a constant to the
// start-address field (16-byte units, no carry out of it: shared memory < 256 KB).
//   Q, K: 128-byte swizzled K-major; K step kk at byte (kk / 4) * 16384 + (kk % 4) * 32
//   V:    128-byte swizzled MN-major; K step kk (16 keys) at byte kk * 2048
__device__ __forceinline__ uint64_t att_qk_desc(const uint8_t* t) { return sdesc_sw128(smem_u32(t), 16, 1024); }
__device__ __forceinline__ uint64_t att_v_desc(const uint8_t* t) { return sdesc_sw128(smem_u32(t), 16384, 1024); }
__host__ __device__ constexpr uint64_t att_qk_step(int kk) { return (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2); }
__host__ __device__ constexpr uint64_t att_v_step(int kk) { return (uint64_t)(kk * 128); }

// Tensor maps over q: f16 [Lq][H][128], k, v: f16 [Lk][Hkv][128] as 3-D tensors
// (head dim, head, row) with boxes of 64 x 1 x 128; o: f32 [Lq][H][128]; group = H / Hkv.
// Grid (ceil(Lq / 128), H).  Requires Lk >= 1.  stall != 0 (failure test only): the
// producers issue no copy, so every other role's first wait runs out.
//
// Buffers with two slots (index b = kb & 1 for key block kb): K, V, S (tensor
// memory), P.  Barriers, each completing once per use of its slot:
//   k_full[b], v_full[b]   TMA transaction count of the 32 KB tile
//   k_empty[b]             commit after Q K^T(kb): the K slot may be refilled
//   s_full[b]              the same commit: S(kb) is ready
//   p_full[b]              softmax threads, after P(kb) is in tensor memory (and S(kb)
//                          read, so the S slot may take block kb + 2)
//   o_done[b], v_empty[b]  commit after P V(kb): O holds blocks 0..kb, and the P and
//                          V slots may be refilled
// A wait on "use u of slot b" takes parity (u >> 1) & 1; no barrier can run two uses
// ahead of its slowest waiter, because each next use needs that waiter's own progress.
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, float* __restrict__ o, int Lq, int Lk, int H,
                     int group, int stall) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* const sQ = smem;
    uint8_t* const sK = smem + ATT_TILE;      // two slots
    uint8_t* const sV = smem + 3 * ATT_TILE;  // two slots
    uint64_t* const bars = reinterpret_cast<uint64_t*>(smem + 5 * ATT_TILE);
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
    float* const xval = reinterpret_cast<float*>(smem + 5 * ATT_TILE + 256);  // [2][half][row]

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
            mbar_init(&p_full[b], 32 * ATT_SOFTMAX_WARPS);
            mbar_init(&o_done[b], 1);
        }
        mbar_init(fin, 2);
        fence_mbar_init();
    }
    if (warp == ATT_MMA_WARP) {
        tmem_alloc(tmem_slot, ATT_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    pdl_wait();  // q, k, v may come from the previous kernel on the stream

    if (warp == ATT_K_WARP || warp == ATT_V_WARP) {
        // ---------------------------------------------------------------- TMA producers
        const bool is_k = warp == ATT_K_WARP;
        const int n_prod = stall ? 0 : nkb;  // stall: no copy at all (failure test)
        if (is_k && !stall) {
            if (lane == 0) mbar_arrive_expect_tx(q_full, ATT_TILE);
            __syncwarp();
            att_tma_tile(sQ, &tq, h, q0, q_full, lane);
        }
        uint64_t* const full = is_k ? k_full : v_full;
        uint64_t* const empty = is_k ? k_empty : v_empty;
        const CUtensorMap* const tmap = is_k ? &tk : &tv;
        uint8_t* const dst = is_k ? sK : sV;
        int issued = 0;
        for (int kb = 0; kb < n_prod; kb++) {
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
            if (is_k && !stall) drain_wait(q_full, 0);
        }
        __syncwarp();
    } else if (warp == ATT_MMA_WARP) {
        // ---------------------------------------------------------------- Q K^T issue
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_f16(ATT_BQ, ATT_BK);
            const uint64_t dq = att_qk_desc(sQ), dk0 = att_qk_desc(sK), dk1 = att_qk_desc(sK + ATT_TILE);
            bool ok = att_wait(q_full, 0);
            for (int kb = 0; ok && kb < nkb; kb++) {
                const int b = kb & 1;
                // S slot b was last read by the softmax of block kb - 2 (P(kb - 2) marks it)
                if (!att_wait(&k_full[b], (kb >> 1) & 1)) break;
                if (kb >= 2 && !att_wait(&p_full[b], ((kb - 2) >> 1) & 1)) break;
                tc_fence_after();
                // S[b] = Q K^T for key block kb: 8 steps of K = 16 along the head dimension.
                const uint32_t d = tm + b * ATT_BK;
                const uint64_t dk = b ? dk1 : dk0;
                mma_f16_ss(d, dq, dk, ID_S, 0);
#pragma unroll
                for (int kk = 1; kk < ATT_DH / 16; kk++)
                    mma_f16_ss(d, dq + att_qk_step(kk), dk + att_qk_step(kk), ID_S, 1);
                tc_commit(&s_full[b]);
                tc_commit(&k_empty[b]);
            }
            // Every MMA issued above completes before the tensor memory is released,
            // also when a wait ran out.
            tc_commit(fin);
            drain_wait(fin, 0);
        }
        __syncwarp();
    } else if (warp == ATT_PV_WARP) {
        // ---------------------------------------------------------------- P V issue
        if (lane == 0) {
            constexpr uint32_t ID_O = idesc_f16(ATT_BQ, ATT_DH) | (1u << 16);  // B (V) MN-major
            const uint64_t dv0 = att_v_desc(sV), dv1 = att_v_desc(sV + ATT_TILE);
            for (int kb = 0; kb < nkb; kb++) {
                const int b = kb & 1;
                if (!att_wait(&p_full[b], (kb >> 1) & 1) || !att_wait(&v_full[b], (kb >> 1) & 1)) break;
                tc_fence_after();
                // O += P V: 8 steps of K = 16 keys (P from tensor memory, 8 columns a step).
                const uint32_t pa = tm + ATT_TM_P + 64 * b;
                const uint64_t dv = b ? dv1 : dv0;
                mma_f16_ts(tm + ATT_TM_O, pa, dv, ID_O, kb > 0);
#pragma unroll
                for (int kk = 1; kk < ATT_BK / 16; kk++)
                    mma_f16_ts(tm + ATT_TM_O, pa + 8 * kk, dv + att_v_step(kk), ID_O, 1);
                tc_commit(&o_done[b]);
                tc_commit(&v_empty[b]);
            }
            tc_commit(fin);
            drain_wait(fin, 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax, output
        const int qd = warp & 3, hf = warp >> 2;
        const int row = 32 * qd + lane;  // query q0 + row, tensor-memory lane row
        const int c0 = 64 * hf;          // this half's key columns of S, head-dim columns of O
        const uint32_t tl = tm + ((uint32_t)(32 * qd) << 16);
        // Swap x with the thread of the other half that owns the same row, at exchange u,
        // through named barrier 1 + qd of the quadrant's two warps.  The barrier also
        // ANDs the two warps' ok flags, so a wait that ran out in either warp stops
        // both at the same exchange: neither is left waiting at the barrier.
        auto swap = [&](int u, float x, float& other, bool ok_in) -> bool {
            xval[((u & 1) * 2 + hf) * 128 + row] = x;
            if (!named_barrier_and(1 + qd, 64, ok_in)) return false;
            other = xval[((u & 1) * 2 + (hf ^ 1)) * 128 + row];
            return true;
        };
        float m = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int kb = 0; kb < nkb; kb++) {
            const int b = kb & 1;
            ok = ok && __all_sync(~0u, att_wait(&s_full[b], (kb >> 1) & 1));  // ok is warp-uniform
            uint32_t sr[64];
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 4; j++) tmem_ld16(tl + b * ATT_BK + c0 + 16 * j, sr + 16 * j);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int j = 0; j < 64; j++) sr[j] = 0u;
            }
            // half-block maximum over the valid keys (eight independent chains); -inf
            // when this half lies past Lk
            const int kvalid = Lk - kb * ATT_BK - c0;
            float mx[8];
#pragma unroll
            for (int e = 0; e < 8; e++) mx[e] = -INFINITY;
            if (kvalid >= 64) {  // uniform across the CTA: no masking
#pragma unroll
                for (int j = 0; j < 64; j++) mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(sr[j]));
            } else {
#pragma unroll
                for (int j = 0; j < 64; j++) {
                    const float x = j < kvalid ? __uint_as_float(sr[j]) : -INFINITY;
                    sr[j] = __float_as_uint(x);
                    mx[j & 7] = fmaxf(mx[j & 7], x);
                }
            }
            const float hm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            float om;
            if (!swap(kb, hm, om, ok)) {
                ok = false;
                break;
            }
            const float mc = fmaxf(hm, om) * ATT_C;  // finite: the block has a valid key
            const bool raise = kb == 0 || mc > m + ATT_RESCALE_LOG2;
            const float m_new = raise ? mc : m;
            // P(kb) = 2^(s c - m_new) in f16 pairs; l sums the unrounded weights.
            uint32_t pk[32];
            float ps[8];
#pragma unroll
            for (int e = 0; e < 8; e++) ps[e] = 0.0f;
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
                const float p0 = att_ex2(fmaf(__uint_as_float(sr[j]), ATT_C, -m_new));
                const float p1 = att_ex2(fmaf(__uint_as_float(sr[j + 1]), ATT_C, -m_new));
                ps[(j >> 1) & 7] += p0 + p1;
                const __half2 hp = __floats2half2_rn(p0, p1);
                pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&hp);
            }
            const float ls = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            // After a wait below runs out, the loop goes on to the next exchange (where
            // both warps stop) without touching tensor memory or the P slot.
            if (kb >= 2) {
                // P V(kb - 2) has read this P slot
                ok = __all_sync(~0u, att_wait(&o_done[b], ((kb - 2) >> 1) & 1));
                if (!ok) continue;
                tc_fence_after();
            }
            if (kb >= 1 && __any_sync(~0u, raise)) {
                // O must hold blocks 0..kb-1 before it is rescaled to the new maximum
                ok = __all_sync(~0u, att_wait(&o_done[b ^ 1], ((kb - 1) >> 1) & 1));
                if (!ok) continue;
                tc_fence_after();
                const float alpha = raise ? att_ex2(m - m_new) : 1.0f;
                l *= alpha;
#pragma unroll 1
                for (int j = 0; j < 4; j++) {
                    uint32_t t[16];
                    tmem_ld16(tl + ATT_TM_O + c0 + 16 * j, t);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e++) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
                    tmem_st16(tl + ATT_TM_O + c0 + 16 * j, t);
                }
                tmem_wait_st();
            }
            l += ls;
            m = m_new;
            // this half's 64 keys = 32 columns of the P slot
            const uint32_t pt = tl + ATT_TM_P + 64 * b + 32 * hf;
            tmem_st16(pt, pk);
            tmem_st16(pt + 16, pk + 16);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[b]);
        }
        // Both warps of the quadrant reach the final exchange: either both left the
        // loop at the same exchange, or both finished it.
        if (ok) ok = __all_sync(~0u, att_wait(&o_done[(nkb - 1) & 1], ((nkb - 1) >> 1) & 1));
        float lo = 0.0f;
        ok = swap(nkb, l, lo, ok);
        if (ok) {
            tc_fence_after();
            const int qi = q0 + row;
            const float inv = 1.0f / (l + lo);
            float* dst = o + ((int64_t)qi * H + h) * ATT_DH + c0;
#pragma unroll 1
            for (int j = 0; j < 4; j++) {
                uint32_t t[16];
                tmem_ld16(tl + ATT_TM_O + c0 + 16 * j, t);
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
    if (warp == ATT_MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tm, ATT_TM_COLS);
    }
}


// ------------------------------------------------------------------------------------
// Two query tiles per CTA ("ping-pong"), for grids of more than one wave.
//
// One CTA per (two query tiles of 128 rows, head), 14 warps, key blocks of 64:
//   warp 9      TMA producer of both Q tiles (once) and of K key blocks (four slots of
//               64 keys); warp 10 the same for V
//   warps 8, 11 one thread each issues S_t(kb) = Q_t K(kb)^T (128 x 64) for query tile
//               0 / tile 1 into one of the tile's two S slots (warp 8 also owns tensor
//               memory); so the tensor core computes the next block's scores while the
//               softmax works on this one
//   warps 12,13 one thread each issues O_t += P_t(kb) V(kb) for tile 0 / tile 1 once
//               the softmax has written P_t(kb) over the first 32 columns of its S slot
//               (the first two K steps as soon as the first 32 keys are in; the slot is
//               reused by S_t(kb + 2) only after that P V has completed).  One
//               thread issues an MMA only every ~55 cycles, so the four streams have a
//               thread each.
//   warps 0-3   softmax of tile 0, warps 4-7 of tile 1; thread = query row = tensor-
//               memory lane 32 (w % 4) + lane, all 64 key columns of the block in
//               registers: block maximum, running maximum m (raised, with O_t and l
//               rescaled once P V(kb - 1) is complete, only when a block maximum exceeds
//               it by more than 8 binades), P = 2^(S c - m) rounded to f16, the running
//               sum l; at the end O_t / l is stored.  Warps w and w + 4 share a sub-
//               partition and its special-function unit; they take turns at the
//               exponentials (tile 0 of block kb, tile 1 of block kb, tile 0 of block
//               kb + 1, ...; each hands over half way through its block), so that each
//               one's loads, maxima and stores run while the other's exponentials keep
//               the unit busy.
// K and V blocks are shared by the two tiles (each slot is released by the commits of
// both issuers): each block crosses from L2 once per 256 queries.
// Tensor memory: O_t at columns 256 t .. 256 t + 127, S slot s of tile t at
// 256 t + 128 + 64 s (64 columns; P in the first 32 as f16 pairs).  A CTA whose
// second tile lies past Lq runs the first one only.
// Shared memory: Q_t as in the one-tile kernel (32 KB each); K and V slots of two TMA
// boxes of 64 head-dim values x 64 keys (8 KB each, 128-byte swizzle): K-major for K
// (second box at +8 KB), MN-major for V (the second 64 head-dim columns at +8 KB, 1024
// bytes per 8 keys).
constexpr int ATT_PP_S0_WARP = 8;  // issues tile 0's Q K^T; owns tensor memory
constexpr int ATT_PP_K_WARP = 9;
constexpr int ATT_PP_V_WARP = 10;
constexpr int ATT_PP_S1_WARP = 11;   // issues tile 1's Q K^T
constexpr int ATT_PP_PV0_WARP = 12;  // issues tile 0's P V
constexpr int ATT_PP_PV1_WARP = 13;  // issues tile 1's P V
constexpr int ATT_PP_THREADS = 32 * 14;
constexpr int ATT_PP_BQ = 2 * ATT_BQ;  // queries per CTA
constexpr int ATT_PP_BK = 64;          // keys per block
constexpr int ATT_PP_SLOTS = 4;        // K and V slots
constexpr int ATT_PP_KV = ATT_PP_BK * ATT_DH * 2;  // one K or V block, 16 KB
// Q x2, K x4, V x4, barriers and tensor-memory address
constexpr size_t ATT_PP_SMEM = 2 * (size_t)ATT_TILE + 2 * ATT_PP_SLOTS * (size_t)ATT_PP_KV + 512;

// Query tiles per CTA for a grid over Lq queries and H heads on a device of `sms` SMs:
// two when one tile per CTA would need more than one wave of CTAs, else one.
__host__ __device__ constexpr int att_tiles_per_cta(int64_t Lq, int64_t H, int sms) {
    return ((Lq + ATT_BQ - 1) / ATT_BQ) * H > sms ? 2 : 1;
}

// K step kk of a 64-key K block (second head-dim box at +8 KB), in 16-byte units.
__host__ __device__ constexpr uint64_t att_k64_step(int kk) { return (uint64_t)((kk >> 2) * 512 + (kk & 3) * 2); }

// Same arguments and grid rows (y = head) as attention_kernel, with K and V maps of
// 64-row boxes; grid x = ceil(Lq / 256).
// Barriers (tile t, S slot s = kb & 1, K/V slot v = kb & 3 for key block kb):
//   q_full[t]                   TMA transaction count of Q_t
//   k_full[v], v_full[v]        TMA transaction count of the 16 KB block
//   k_empty[v], v_empty[v]      one commit per active tile, after Q_t K^T(kb) / P_t V(kb)
//   s_full[t][s]                commit after Q_t K^T(kb)
//   p_half[t][s], p_full[t][s]  the tile's four softmax warps (one arrival each), after
//                               the first 32 keys of P_t(kb) / all of it
//   o_done[t][s]                commit after P_t V(kb)
//   ex[q][t]                    lane 0 of tile t's softmax warp of quadrant q, half way
//                               through its exponentials of block kb (the turn passes to
//                               the other tile)
// A barrier of slot kb % n completes once per use u = kb / n and a wait takes parity
// u & 1: (kb >> 1) & 1 for the tile barriers, (kb >> 2) & 1 for the K/V slots.  No
// barrier runs two uses ahead of a waiter, because its next use needs that waiter's own
// progress.
__global__ void __launch_bounds__(ATT_PP_THREADS, 1)
    attention_pp_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, float* __restrict__ o, int Lq, int Lk, int H,
                        int group, int stall) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* const sQ = smem;                                    // two tiles
    uint8_t* const sK = smem + 2 * ATT_TILE;                     // four slots
    uint8_t* const sV = sK + ATT_PP_SLOTS * ATT_PP_KV;           // four slots
    uint64_t* const bars = reinterpret_cast<uint64_t*>(sV + ATT_PP_SLOTS * ATT_PP_KV);
    uint64_t* const q_full = bars;       // [2]
    uint64_t* const k_full = bars + 2;   // [4]
    uint64_t* const v_full = bars + 6;   // [4]
    uint64_t* const k_empty = bars + 10; // [4]
    uint64_t* const v_empty = bars + 14; // [4]
    uint64_t* const s_full = bars + 18;  // [2][2]
    uint64_t* const p_full = bars + 22;  // [2][2]
    uint64_t* const o_done = bars + 26;  // [2][2]
    uint64_t* const fin = bars + 30;
    uint64_t* const ex = bars + 31;      // [4][2]
    uint64_t* const p_half = bars + 39;  // [2][2]
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(bars + 43);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * ATT_PP_BQ, h = blockIdx.y, hk = h / group;
    const int ntiles = Lq - q0 > ATT_BQ ? 2 : 1;
    const int nkb = (Lk + ATT_PP_BK - 1) / ATT_PP_BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; i++) mbar_init(&q_full[i], 1);
        for (int i = 0; i < ATT_PP_SLOTS; i++) {
            mbar_init(&k_full[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&k_empty[i], ntiles);
            mbar_init(&v_empty[i], ntiles);
        }
        for (int i = 0; i < 4; i++) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&p_half[i], 4);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(fin, 4);
        for (int i = 0; i < 8; i++) mbar_init(&ex[i], 1);
        fence_mbar_init();
    }
    if (warp == ATT_PP_S0_WARP) {
        tmem_alloc(tmem_slot, ATT_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    pdl_wait();  // q, k, v may come from the previous kernel on the stream

    if (warp == ATT_PP_K_WARP || warp == ATT_PP_V_WARP) {
        // ---------------------------------------------------------------- TMA producers
        const bool is_k = warp == ATT_PP_K_WARP;
        const int n_prod = stall ? 0 : nkb;  // stall: no copy at all (failure test)
        if (is_k && !stall) {
            for (int t = 0; t < ntiles; t++) {
                if (lane == 0) mbar_arrive_expect_tx(&q_full[t], ATT_TILE);
                __syncwarp();
                if (lane < 2) tma_load_3d(sQ + t * ATT_TILE + lane * (ATT_TILE / 2), &tq, 64 * lane, h, q0 + t * ATT_BQ,
                                          &q_full[t]);
            }
        }
        uint64_t* const full = is_k ? k_full : v_full;
        uint64_t* const empty = is_k ? k_empty : v_empty;
        const CUtensorMap* const tmap = is_k ? &tk : &tv;
        uint8_t* const dst = is_k ? sK : sV;
        int issued = 0;
        for (int kb = 0; kb < n_prod; kb++) {
            const int v = kb & 3;
            if (kb >= ATT_PP_SLOTS && !__all_sync(~0u, att_wait(&empty[v], ((kb >> 2) - 1) & 1))) break;
            if (lane == 0) mbar_arrive_expect_tx(&full[v], ATT_PP_KV);
            __syncwarp();
            if (lane < 2)
                tma_load_3d(dst + v * ATT_PP_KV + lane * (ATT_PP_KV / 2), tmap, 64 * lane, hk, kb * ATT_PP_BK, &full[v]);
            issued = kb + 1;
        }
        // No copy may still be landing in shared memory when the CTA exits, also when
        // a wait ran out: wait for the last use of each slot (and for the Q tiles).
        if (lane == 0) {
            for (int kb = issued > ATT_PP_SLOTS ? issued - ATT_PP_SLOTS : 0; kb < issued; kb++)
                drain_wait(&full[kb & 3], (kb >> 2) & 1);
            if (is_k && !stall)
                for (int t = 0; t < ntiles; t++) drain_wait(&q_full[t], 0);
        }
        __syncwarp();
    } else if (warp == ATT_PP_S0_WARP || warp == ATT_PP_S1_WARP) {
        // ---------------------------------------------------------------- Q K^T issue, tile t
        const int t = warp == ATT_PP_S0_WARP ? 0 : 1;
        if (lane == 0 && t < ntiles) {
            constexpr uint32_t ID_S = idesc_f16(ATT_BQ, ATT_PP_BK);
            const uint32_t tb = tm + 256 * t;  // O_t; S slots at +128 and +192
            const uint64_t dq = att_qk_desc(sQ + t * ATT_TILE);
            const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
            bool ok = att_wait(&q_full[t], 0);
            for (int kb = 0; ok && kb < nkb; kb++) {
                const int sl = kb & 1, v = kb & 3;
                if (!att_wait(&k_full[v], (kb >> 2) & 1)) break;
                // P V(kb - 2) has read P out of this S slot
                if (kb >= 2 && !att_wait(&o_done[2 * t + sl], ((kb - 2) >> 1) & 1)) break;
                tc_fence_after();
                const uint32_t ds = tb + 128 + 64 * sl;
                const uint64_t dk = dk0 + (uint64_t)(v * (ATT_PP_KV >> 4));
                mma_f16_ss(ds, dq, dk, ID_S, 0);
#pragma unroll
                for (int kk = 1; kk < ATT_DH / 16; kk++)
                    mma_f16_ss(ds, dq + att_qk_step(kk), dk + att_k64_step(kk), ID_S, 1);
                tc_commit(&s_full[2 * t + sl]);
                tc_commit(&k_empty[v]);
            }
        }
        // Every MMA issued above completes before the tensor memory is released, also
        // when a wait ran out (a thread that issued none arrives at once).
        if (lane == 0) {
            tc_commit(fin);
            drain_wait(fin, 0);
        }
        __syncwarp();
    } else if (warp == ATT_PP_PV0_WARP || warp == ATT_PP_PV1_WARP) {
        // ---------------------------------------------------------------- P V issue, tile t
        const int t = warp == ATT_PP_PV0_WARP ? 0 : 1;
        if (lane == 0 && t < ntiles) {
            constexpr uint32_t ID_O = idesc_f16(ATT_BQ, ATT_DH) | (1u << 16);  // B (V) MN-major
            const uint32_t tb = tm + 256 * t;
            const uint64_t dv0 = sdesc_sw128(smem_u32(sV), ATT_PP_KV / 2, 1024);
            for (int kb = 0; kb < nkb; kb++) {
                const int sl = kb & 1, v = kb & 3;
                // O_t += P_t V: 4 steps of K = 16 keys (P from tensor memory, 8 columns a
                // step), the first two as soon as the first half of P is in.
                if (!att_wait(&p_half[2 * t + sl], (kb >> 1) & 1) || !att_wait(&v_full[v], (kb >> 2) & 1)) break;
                tc_fence_after();
                const uint32_t pa = tb + 128 + 64 * sl;
                const uint64_t dv = dv0 + (uint64_t)(v * (ATT_PP_KV >> 4));
                mma_f16_ts(tb, pa, dv, ID_O, kb > 0);
                mma_f16_ts(tb, pa + 8, dv + att_v_step(1), ID_O, 1);
                if (!att_wait(&p_full[2 * t + sl], (kb >> 1) & 1)) break;
                tc_fence_after();
                mma_f16_ts(tb, pa + 16, dv + att_v_step(2), ID_O, 1);
                mma_f16_ts(tb, pa + 24, dv + att_v_step(3), ID_O, 1);
                tc_commit(&o_done[2 * t + sl]);
                tc_commit(&v_empty[v]);
            }
        }
        if (lane == 0) {
            tc_commit(fin);
            drain_wait(fin, 0);
        }
        __syncwarp();
    } else if ((warp >> 2) < ntiles) {
        // ---------------------------------------------------------------- softmax, output
        const int t = warp >> 2, qd = warp & 3;
        const int row = 32 * qd + lane;  // query q0 + 128 t + row, tensor-memory lane row
        const uint32_t tb = tm + ((uint32_t)(32 * qd) << 16) + 256 * t;  // this warp's lanes of O_t
        float m = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int kb = 0; kb < nkb; kb++) {
            const int sl = kb & 1;
            ok = __all_sync(~0u, att_wait(&s_full[2 * t + sl], (kb >> 1) & 1));  // warp-uniform
            if (!ok) break;
            tc_fence_after();
            const uint32_t ts = tb + 128 + 64 * sl;
            uint32_t sr[ATT_PP_BK];
            // S in two halves: the maximum of the first runs while the second loads.
            tmem_ld16(ts, sr);
            tmem_ld16(ts + 16, sr + 16);
            tmem_wait_ld();
            tmem_ld16(ts + 32, sr + 32);
            tmem_ld16(ts + 48, sr + 48);
            // block maximum over the valid keys (eight independent chains of 3-input max)
            const int kvalid = Lk - kb * ATT_PP_BK;
            float mx[8];
#pragma unroll
            for (int e = 0; e < 8; e++) mx[e] = -INFINITY;
            if (kvalid >= ATT_PP_BK) {  // uniform across the CTA: no masking
#pragma unroll
                for (int j = 0; j < ATT_PP_BK / 2; j += 2)
                    mx[(j >> 1) & 7] = max3f(mx[(j >> 1) & 7], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                tmem_wait_ld();
#pragma unroll
                for (int j = ATT_PP_BK / 2; j < ATT_PP_BK; j += 2)
                    mx[(j >> 1) & 7] = max3f(mx[(j >> 1) & 7], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
            } else {
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < ATT_PP_BK; j++) {
                    const float x = j < kvalid ? __uint_as_float(sr[j]) : -INFINITY;
                    sr[j] = __float_as_uint(x);
                    mx[j & 7] = fmaxf(mx[j & 7], x);
                }
            }
            const float mc = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
                             ATT_C;  // finite: the block has a valid key
            const bool raise = kb == 0 || mc > m + ATT_RESCALE_LOG2;
            const float m_new = raise ? mc : m;
            if (kb >= 1 && __any_sync(~0u, raise)) {
                // O_t must hold blocks 0..kb-1 before it is rescaled to the new maximum
                ok = __all_sync(~0u, att_wait(&o_done[2 * t + (sl ^ 1)], ((kb - 1) >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
                const float alpha = raise ? att_ex2(m - m_new) : 1.0f;
                l *= alpha;
#pragma unroll 1
                for (int j = 0; j < ATT_DH / 16; j++) {
                    uint32_t r[16];
                    tmem_ld16(tb + 16 * j, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e++) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                    tmem_st16(tb + 16 * j, r);
                }
            }
            m = m_new;
            // this sub-partition's turn at the exponentials: tile 1 after tile 0 of the same
            // block, tile 0 after tile 1 of the previous block
            if (ntiles == 2 && (t == 1 || kb >= 1)) {
                ok = __all_sync(~0u, att_wait(&ex[2 * qd + (t ^ 1)], (t == 1 ? kb : kb - 1) & 1));
                if (!ok) break;
            }
            // P(kb) = 2^(s c - m) in f16 pairs over the slot's first 32 columns; l sums
            // the unrounded weights.
            float ps[8];
#pragma unroll
            for (int e = 0; e < 8; e++) ps[e] = 0.0f;
#pragma unroll
            for (int c = 0; c < ATT_PP_BK / 32; c++) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; e++) {
                    const float p0 = att_ex2(fmaf(__uint_as_float(sr[32 * c + 2 * e]), ATT_C, -m));
                    const float p1 = att_ex2(fmaf(__uint_as_float(sr[32 * c + 2 * e + 1]), ATT_C, -m));
                    ps[e & 7] += p0 + p1;
                    const __half2 hp = __floats2half2_rn(p0, p1);
                    pk[e] = *reinterpret_cast<const uint32_t*>(&hp);
                }
                tmem_st16(ts + 16 * c, pk);
                if (c == 0) {
                    // half way: P V may start on these keys, and the other tile may start
                    // its exponentials
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&p_half[2 * t + sl]);
                        mbar_arrive(&ex[2 * qd + t]);
                    }
                }
            }
            l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[2 * t + sl]);  // one arrival per warp
        }
        if (ok) ok = __all_sync(~0u, att_wait(&o_done[2 * t + ((nkb - 1) & 1)], ((nkb - 1) >> 1) & 1));
        if (ok) {
            tc_fence_after();
            const int qi = q0 + ATT_BQ * t + row;
            const float inv = 1.0f / l;
            float* dst = o + ((int64_t)qi * H + h) * ATT_DH;
#pragma unroll 1
            for (int j = 0; j < ATT_DH / 16; j++) {
                uint32_t r[16];
                tmem_ld16(tb + 16 * j, r);
                tmem_wait_ld();
                if (qi < Lq) {
#pragma unroll
                    for (int e = 0; e < 4; e++)
                        reinterpret_cast<float4*>(dst + 16 * j)[e] =
                            make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                                        __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == ATT_PP_S0_WARP) {
        tc_fence_after();
        tmem_dealloc(tm, ATT_TM_COLS);
    }
}

}  // namespace dllm
