// Q4_K / Q6_K x int8 projection GEMM on the sm_100a tensor cores.
//
// What one output element is (mojo-dllm Architecture page, "A forward pass", step 2,
// and "Source map", gpu/kernels.mojo row: an int8 tensor-core GEMM over Q4_K / Q6_K
// blocks):
//   out[m][n] = sum_sb da[m][sb] * (d[n][sb] * S - dmin[n][sb] * Smin)      (Q4_K)
//   out[m][n] = sum_sb da[m][sb] *  d[n][sb] * S                           (Q6_K)
//   S    = sum_k (q_k * sc_j(k)) * a_k      (Q6_K: (q_k - 32) * sc_j(k))
//   Smin = sum_j m_j * sum32_j(a)
//
// How it is computed.  The tensor core multiplies 8-bit operands, and q*sc needs
// 10 bits (Q4_K) or 13 bits (Q6_K), so the weight operand is split into two 8-bit
// planes whose integer results are recombined exactly:
//   Q4_K: sc = lo3 + 8*hi3 (3 bits each); plane 0 = q*lo3, plane 1 = q*hi3, both in
//         0..105 (u8).  S = P0 + 8*P1.
//   Q6_K: v = (q-32)*sc + 32896 lies in [28800, 36992]; plane 0 = (v & 255) - 128,
//         plane 1 = (v >> 8) - 128 (both s8), and plane0 + 256*plane1 = (q-32)*sc.
// The min term of Q4_K is two more MMAs per super-block with the mins m_j (u8) as A
// and the per-32 activation sums, split into an unsigned low byte and a signed high
// byte, as B: Smin = Ml + 256*Mh.
//
// Every integer accumulator stays within 2^22 in magnitude.  Tensor memory is
// preset to the bit pattern of 1.5*2^23 before each super-block, so the int32 the
// MMAs leave there, read as an f32, is exactly 1.5*2^23 + value; the epilogue turns
// it into floats with one FFMA and one FADD per pair of accumulators, with no
// integer-to-float conversion instruction.
//
// Roles (16 warps, one CTA per SM, persistent over work units):
//   warp 0      producer: bulk copies of weight tiles and activation tiles into
//               shared-memory rings (or a gather of requested rows)
//   warp 1      tensor-memory allocation, and one thread issuing every tcgen05.mma
//   warps 4-7   unpack: thread = weight row; decode the super-block, build the two
//               weight planes for each K-step of 32 and store them into tensor
//               memory (the A operand), plus the mins and the f32 d/dmin
//   warps 8-15  epilogue: two warps per tensor-memory lane quadrant, each on half of
//               the token columns; per super-block, read the integer accumulators,
//               preset them again, and accumulate the f32 result in registers
// A work unit is (128 weight rows, up to 128 canvas rows, all of K).
#pragma once
#include "layout.cuh"

namespace dllm {

constexpr uint32_t MAGIC_BITS = 0x4B400000u;  // 1.5 * 2^23
constexpr float MAGIC = 12582912.0f;
constexpr int GEMM_THREADS = 512;
constexpr int UNIT_TOKENS = 128;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s

template <int QT>
struct GemmCfg;
template <>
struct GemmCfg<12> {  // Q4_K
    static constexpr int TILE = Q4K_TILE;
    static constexpr int NTOK = 32;  // token columns per MMA and per accumulator
    static constexpr int NACC = 4;   // P0, P1, Ml, Mh
    static constexpr int W_STAGES = 4;
    static constexpr int B_STAGES = 8;
    static constexpr int B_Q = NTOK * 256;
    static constexpr int B_SUMS = NTOK * 16 + 128;
    static constexpr int B_STAGE = B_Q + B_SUMS + NTOK * 4;
};
template <>
struct GemmCfg<14> {  // Q6_K
    static constexpr int TILE = Q6K_TILE;
    static constexpr int NTOK = 64;
    static constexpr int NACC = 2;  // P0, P1
    static constexpr int W_STAGES = 3;
    static constexpr int B_STAGES = 4;
    static constexpr int B_Q = NTOK * 256;
    static constexpr int B_SUMS = 0;
    static constexpr int B_STAGE = B_Q + B_SUMS + NTOK * 4;
};

constexpr int S_SLOTS = 4;  // d/dmin ring (unpack -> epilogue)
constexpr int ACC_SETS = 2;
// tensor-memory columns
constexpr uint32_t TM_A = 0;       // 8 K-step slots x 16 columns (plane 0 | plane 1)
constexpr uint32_t TM_AMIN = 128;  // 2 buffers x 16 columns (Ml-A | Mh-A)
constexpr uint32_t TM_ACC = 160;   // ACC_SETS x NACC x NTOK columns
constexpr uint32_t TM_COLS = 512;

struct Segment {
    const uint8_t* w;   // repacked weights
    float* out;
    int64_t ldo;
    int32_t tile0;      // first global n-tile of this segment
};

struct GemmArgs {
    Segment seg[3];
    int nseg;
    int32_t n_tiles;    // total 128-row tiles over all segments
    int32_t nsb;        // K / 256
    const int8_t* q;    // tiled activations of the source canvas
    const float* scale;
    const uint8_t* sums;
    int64_t M;          // source canvas rows
    int64_t Mp;         // M rounded up to 16 (the layout's row count)
    const int32_t* rows;  // nullable
    int32_t n_rows;
    int32_t n_st;       // token super-tiles per n-tile
    int32_t mu;         // tokens per super-tile (multiple of 16)
    int64_t m_out;      // output rows (M or n_rows)
    int32_t* dbg_S;     // debug: integer outputs instead of f32 (nullable)
    int32_t* dbg_Smin;
    int64_t dbg_N;
};

struct GemmShared {
    uint64_t w_full[8], w_empty[8];
    uint64_t b_full[8], b_empty[8];
    uint64_t a_full[8], a_empty[8];
    uint64_t amin_full[2], amin_empty[2];
    uint64_t s_full[S_SLOTS], s_empty[S_SLOTS];
    uint64_t acc_full[ACC_SETS], acc_empty[ACC_SETS];
    uint64_t final_bar;
    uint32_t tmem_base;
    volatile int abort_flag;
    float2 dd[S_SLOTS][TROWS];
};

// Bounded wait on an mbarrier phase; false if this CTA is aborting.  Raises the
// abort flag and the device error word when the limit runs out.
__device__ __forceinline__ bool wait_bar(GemmShared& sh, uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (sh.abort_flag) return false;
        if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            sh.abort_flag = 1;
            set_err(ERR_TIMEOUT);
            return false;
        }
    }
}
// Warp-uniform variant: every lane waits, and the warp agrees on the outcome.
__device__ __forceinline__ bool wait_bar_warp(GemmShared& sh, uint64_t* bar, uint32_t parity) {
    const bool ok = wait_bar(sh, bar, parity);
    return __all_sync(0xffffffffu, ok);
}

struct Unit {
    int seg;
    int64_t tile;   // tile index inside the segment
    int64_t m0;     // first token of the super-tile (in the gathered numbering when rows)
    int32_t len;    // tokens in the super-tile (multiple of 16)
};

__device__ __forceinline__ Unit unit_of(const GemmArgs& a, int64_t u) {
    Unit r;
    const int64_t nt = u / a.n_st;
    const int32_t st = (int32_t)(u % a.n_st);
    r.seg = 0;
    if (a.nseg > 1 && nt >= a.seg[1].tile0) r.seg = 1;
    if (a.nseg > 2 && nt >= a.seg[2].tile0) r.seg = 2;
    r.tile = nt - a.seg[r.seg].tile0;
    r.m0 = (int64_t)st * a.mu;
    const int64_t rows_total = a.rows ? round_up(a.n_rows, 16) : a.Mp;
    r.len = (int32_t)min((int64_t)a.mu, rows_total - r.m0);
    return r;
}

template <int QT, bool DBG>
__global__ void __launch_bounds__(GEMM_THREADS, 1) qgemm_kernel(const __grid_constant__ GemmArgs args) {
    using C = GemmCfg<QT>;
    constexpr int NTOK = C::NTOK;
    constexpr int TMAX = UNIT_TOKENS / NTOK;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* w_stage = smem_raw;
    uint8_t* b_stage = w_stage + C::W_STAGES * C::TILE;
    GemmShared& sh = *reinterpret_cast<GemmShared*>(b_stage + C::B_STAGES * C::B_STAGE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_units = (int64_t)args.n_tiles * args.n_st;
    const int nsb = args.nsb;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::W_STAGES; i++) { mbar_init(&sh.w_full[i], 1); mbar_init(&sh.w_empty[i], 128); }
        for (int i = 0; i < C::B_STAGES; i++) { mbar_init(&sh.b_full[i], 1); mbar_init(&sh.b_empty[i], 1 + 256); }
        for (int i = 0; i < 8; i++) { mbar_init(&sh.a_full[i], 128); mbar_init(&sh.a_empty[i], 1); }
        for (int i = 0; i < 2; i++) { mbar_init(&sh.amin_full[i], 128); mbar_init(&sh.amin_empty[i], 1); }
        for (int i = 0; i < S_SLOTS; i++) { mbar_init(&sh.s_full[i], 128); mbar_init(&sh.s_empty[i], 256); }
        for (int i = 0; i < ACC_SETS; i++) { mbar_init(&sh.acc_full[i], 1); mbar_init(&sh.acc_empty[i], 256); }
        mbar_init(&sh.final_bar, 1);
        sh.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    if (warp == 0) {
        // ============================================================ producer
        uint32_t ws = 0, wph = 0, bs = 0, bph = 0;
        uint32_t w_issued_ph[C::W_STAGES], b_issued_ph[C::B_STAGES];
        bool w_issued[C::W_STAGES], b_issued[C::B_STAGES];
        for (int i = 0; i < C::W_STAGES; i++) w_issued[i] = false;
        for (int i = 0; i < C::B_STAGES; i++) b_issued[i] = false;
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_a = policy_evict_last();
        for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
            const Unit un = unit_of(args, u);
            const uint8_t* wt = args.seg[un.seg].w + (size_t)un.tile * nsb * C::TILE;
            const int T = (un.len + NTOK - 1) / NTOK;
            for (int s = 0; s < nsb; s++) {
                if (!wait_bar_warp(sh, &sh.w_empty[ws], wph ^ 1)) goto done;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sh.w_full[ws], C::TILE);
                    bulk_g2s_hint(w_stage + ws * C::TILE, wt + (size_t)s * C::TILE, C::TILE, &sh.w_full[ws], pol_w);
                }
                w_issued[ws] = true;
                w_issued_ph[ws] = wph;
                if (++ws == C::W_STAGES) { ws = 0; wph ^= 1; }
                for (int tt = 0; tt < T; tt++) {
                    const int64_t t0 = un.m0 + (int64_t)tt * NTOK;
                    const int ntok = min(NTOK, un.len - tt * NTOK);
                    if (!wait_bar_warp(sh, &sh.b_empty[bs], bph ^ 1)) goto done;
                    uint8_t* st = b_stage + bs * C::B_STAGE;
                    if (args.rows == nullptr) {
                        if (lane == 0) {
                            const uint32_t bytes = ntok * 256 + (C::B_SUMS ? ntok * 16 : 0) + ntok * 4;
                            mbar_arrive_expect_tx(&sh.b_full[bs], bytes);
                            bulk_g2s_hint(st, args.q + ((size_t)s * args.Mp + t0) * 256, ntok * 256,
                                          &sh.b_full[bs], pol_a);
                            if (C::B_SUMS)
                                bulk_g2s_hint(st + C::B_Q, args.sums + ((size_t)s * args.Mp + t0) * 16, ntok * 16,
                                              &sh.b_full[bs], pol_a);
                            bulk_g2s_hint(st + C::B_Q + C::B_SUMS, args.scale + (size_t)s * args.Mp + t0, ntok * 4,
                                          &sh.b_full[bs], pol_a);
                        }
                    } else {
                        // gather requested rows: 16-byte chunks, canvas row rows[i]
                        for (int idx = lane; idx < ntok * 18; idx += 32) {
                            const int i = idx / 18, c = idx % 18;  // c < 16: q chunk; 16: sums; 17: scale
                            const int64_t gi = t0 + i;
                            int64_t m = -1;
                            if (gi < args.n_rows) {
                                m = args.rows[gi];
                                if (m < 0 || m >= args.M) {
                                    if (c == 0) set_err(ERR_ROW_RANGE);
                                    m = -1;
                                }
                            }
                            if (c < 16) {
                                uint4 v = make_uint4(0, 0, 0, 0);
                                if (m >= 0)
                                    v = *reinterpret_cast<const uint4*>(
                                        args.q + (((size_t)s * (args.Mp / 8) + m / 8) * 16 + c) * 128 + (m % 8) * 16);
                                *reinterpret_cast<uint4*>(st + ((i / 8) * 16 + c) * 128 + (i % 8) * 16) = v;
                            } else if (c == 16) {
                                if (C::B_SUMS) {
                                    uint4 v = make_uint4(0, 0, 0, 0);
                                    if (m >= 0)
                                        v = *reinterpret_cast<const uint4*>(args.sums + ((size_t)s * args.Mp + m) * 16);
                                    *reinterpret_cast<uint4*>(st + C::B_Q + i * 16) = v;
                                }
                            } else {
                                float v = 0.0f;
                                if (m >= 0) v = args.scale[(size_t)s * args.Mp + m];
                                reinterpret_cast<float*>(st + C::B_Q + C::B_SUMS)[i] = v;
                            }
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sh.b_full[bs]);
                    }
                    b_issued[bs] = args.rows == nullptr;
                    b_issued_ph[bs] = bph;
                    if (++bs == C::B_STAGES) { bs = 0; bph ^= 1; }
                }
            }
        }
    done:
        // never leave with bulk copies in flight into this CTA's shared memory
        if (sh.abort_flag) {
            for (int i = 0; i < C::W_STAGES; i++)
                if (w_issued[i]) (void)wait_bar(sh, &sh.w_full[i], w_issued_ph[i]);
            for (int i = 0; i < C::B_STAGES; i++)
                if (b_issued[i]) (void)wait_bar(sh, &sh.b_full[i], b_issued_ph[i]);
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            uint32_t bs = 0, bph = 0, r = 0, rph = 0, ab = 0, sbc = 0;
            uint32_t amin_ph[2] = {0, 0};
            for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
                const Unit un = unit_of(args, u);
                const int T = (un.len + NTOK - 1) / NTOK;
                for (int s = 0; s < nsb; s++, sbc++) {
                    for (int tt = 0; tt < T; tt++) {
                        const int ntok = min(NTOK, un.len - tt * NTOK);
                        if (!wait_bar(sh, &sh.b_full[bs], bph)) goto mma_done;
                        if (!wait_bar(sh, &sh.acc_empty[r], rph)) goto mma_done;
                        tc_fence_after();
                        const uint32_t st = smem_u32(b_stage + bs * C::B_STAGE);
                        const uint32_t acc = tmem + TM_ACC + r * C::NACC * NTOK;
                        const uint32_t id_p = QT == 12 ? idesc_i8(128, ntok, 0, 1) : idesc_i8(128, ntok, 1, 1);
                        for (int ks = 0; ks < 8; ks++) {
                            if (tt == 0) {
                                if (!wait_bar(sh, &sh.a_full[ks], sbc & 1)) goto mma_done;
                                tc_fence_after();
                            }
                            const uint64_t bd = sdesc_kmajor_noswz(st + 256 * ks, 128, 2048);
                            mma_i8_ts(acc + 0 * NTOK, tmem + TM_A + 16 * ks, bd, id_p, 1);
                            mma_i8_ts(acc + 1 * NTOK, tmem + TM_A + 16 * ks + 8, bd, id_p, 1);
                            if (tt == T - 1) tc_commit(&sh.a_empty[ks]);
                        }
                        if constexpr (QT == 12) {
                            if (tt == 0) {
                                if (!wait_bar(sh, &sh.amin_full[ab], amin_ph[ab])) goto mma_done;
                                tc_fence_after();
                            }
                            const uint64_t bd = sdesc_kmajor_noswz(st + C::B_Q, 128, 128);
                            mma_i8_ts(acc + 2 * NTOK, tmem + TM_AMIN + 16 * ab, bd, idesc_i8(128, ntok, 0, 0), 1);
                            mma_i8_ts(acc + 3 * NTOK, tmem + TM_AMIN + 16 * ab + 8, bd, idesc_i8(128, ntok, 0, 1), 1);
                            if (tt == T - 1) tc_commit(&sh.amin_empty[ab]);
                        }
                        tc_commit(&sh.acc_full[r]);
                        tc_commit(&sh.b_empty[bs]);
                        if (++bs == C::B_STAGES) { bs = 0; bph ^= 1; }
                        if (++r == ACC_SETS) { r = 0; rph ^= 1; }
                    }
                    if (QT == 12) { amin_ph[ab] ^= 1; ab ^= 1; }
                }
            }
        mma_done:
            // every MMA this thread issued has completed before tensor memory is freed
            tc_commit(&sh.final_bar);
            (void)wait_bar(sh, &sh.final_bar, 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ============================================================ unpack
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        uint32_t ws = 0, wph = 0, ss = 0, sph = 0, ab = 0, sbc = 0;
        uint32_t amin_ph[2] = {0, 0};
        for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
            for (int s = 0; s < nsb; s++, sbc++) {
                if (!wait_bar_warp(sh, &sh.w_full[ws], wph)) goto unpack_done;
                const uint8_t* tl = w_stage + ws * C::TILE;
                if constexpr (QT == 12) {
                    // ---- Q4_K: scales, mins, d, dmin of this row
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_SC + 12 * row);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_SC + 12 * row + 4);
                    const uint32_t b2 = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_SC + 12 * row + 8);
                    const uint32_t dm = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_D + 4 * row);
                    uint32_t sc[8], mn[8];
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        sc[j] = (b0 >> (8 * j)) & 63;
                        mn[j] = (b1 >> (8 * j)) & 63;
                        sc[j + 4] = ((b2 >> (8 * j)) & 15) | (((b0 >> (8 * j + 6)) & 3) << 4);
                        mn[j + 4] = ((b2 >> (8 * j + 4)) & 15) | (((b1 >> (8 * j + 6)) & 3) << 4);
                    }
                    const float d = __half2float(__ushort_as_half((unsigned short)(dm & 0xFFFF)));
                    const float dmin = __half2float(__ushort_as_half((unsigned short)(dm >> 16)));
                    if (!wait_bar_warp(sh, &sh.s_empty[ss], sph ^ 1)) goto unpack_done;
                    sh.dd[ss][row] = make_float2(d, -dmin);
                    mbar_arrive(&sh.s_full[ss]);
                    if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
                    // mins as the A operand of the two min-term MMAs
                    if (!wait_bar_warp(sh, &sh.amin_empty[ab], amin_ph[ab] ^ 1)) goto unpack_done;
                    {
                        uint32_t v[16];
#pragma unroll
                        for (int i = 0; i < 16; i++) v[i] = 0;
                        v[0] = mn[0] | (mn[1] << 8) | (mn[2] << 16) | (mn[3] << 24);
                        v[1] = mn[4] | (mn[5] << 8) | (mn[6] << 16) | (mn[7] << 24);
                        v[10] = v[0];
                        v[11] = v[1];
                        tmem_st16(tmem + lane_off + TM_AMIN + 16 * ab, v);
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sh.amin_full[ab]);
                    }
                    amin_ph[ab] ^= 1;
                    ab ^= 1;
                    // weight planes, one K-step (= one sub-block of 32) at a time
#pragma unroll 1
                    for (int c = 0; c < 4; c++) {
                        const uint4 p0 = *reinterpret_cast<const uint4*>(tl + ((2 * c) * TROWS + row) * 16);
                        const uint4 p1 = *reinterpret_cast<const uint4*>(tl + ((2 * c + 1) * TROWS + row) * 16);
                        const uint32_t wv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                        for (int h = 0; h < 2; h++) {
                            const int ks = 2 * c + h;
                            if (!wait_bar_warp(sh, &sh.a_empty[ks], (sbc & 1) ^ 1)) goto unpack_done;
                            const uint32_t lo3 = sc[ks] & 7, hi3 = sc[ks] >> 3;
                            uint32_t v[16];
#pragma unroll
                            for (int i = 0; i < 8; i++) {
                                const uint32_t nib = (wv[i] >> (4 * h)) & 0x0F0F0F0Fu;
                                v[i] = nib * lo3;
                                v[8 + i] = nib * hi3;
                            }
                            tmem_st16(tmem + lane_off + TM_A + 16 * ks, v);
                            tmem_wait_st();
                            tc_fence_before();
                            mbar_arrive(&sh.a_full[ks]);
                        }
                    }
                } else {
                    // ---- Q6_K
                    const uint4 scv = *reinterpret_cast<const uint4*>(tl + Q6K_OFF_SC + 16 * row);
                    const uint32_t scw[4] = {scv.x, scv.y, scv.z, scv.w};
                    const float d = __half2float(
                        __ushort_as_half(*reinterpret_cast<const unsigned short*>(tl + Q6K_OFF_D + 2 * row)));
                    if (!wait_bar_warp(sh, &sh.s_empty[ss], sph ^ 1)) goto unpack_done;
                    sh.dd[ss][row] = make_float2(d, 0.0f);
                    mbar_arrive(&sh.s_full[ss]);
                    if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
#pragma unroll 1
                    for (int ks = 0; ks < 8; ks++) {
                        const int h = ks >> 2, g = ks & 3;
                        const int lp = 2 * (2 * h + (g & 1));  // low-bit piece index
                        const uint4 l0 = *reinterpret_cast<const uint4*>(tl + (lp * TROWS + row) * 16);
                        const uint4 l1 = *reinterpret_cast<const uint4*>(tl + ((lp + 1) * TROWS + row) * 16);
                        const uint4 h0 =
                            *reinterpret_cast<const uint4*>(tl + Q6K_OFF_QH + ((2 * h) * TROWS + row) * 16);
                        const uint4 h1 =
                            *reinterpret_cast<const uint4*>(tl + Q6K_OFF_QH + ((2 * h + 1) * TROWS + row) * 16);
                        const uint32_t lw[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
                        const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                        const int sh_lo = 4 * (g >> 1), sh_hi = 2 * g;
                        const int32_t sca = (int32_t)(int8_t)((scw[ks >> 1] >> (16 * (ks & 1))) & 0xFF);
                        const int32_t scb = (int32_t)(int8_t)((scw[ks >> 1] >> (16 * (ks & 1) + 8)) & 0xFF);
                        const uint32_t adda = (uint32_t)(32896 - 32 * sca) * 0x10001u;
                        const uint32_t addb = (uint32_t)(32896 - 32 * scb) * 0x10001u;
                        if (!wait_bar_warp(sh, &sh.a_empty[ks], (sbc & 1) ^ 1)) goto unpack_done;
                        uint32_t v[16];
#pragma unroll
                        for (int i = 0; i < 8; i++) {
                            const uint32_t qv = ((lw[i] >> sh_lo) & 0x0F0F0F0Fu) | (((hw[i] >> sh_hi) & 0x03030303u) << 4);
                            const int32_t sc = i < 4 ? sca : scb;
                            const uint32_t add = i < 4 ? adda : addb;
                            const uint32_t pa = __byte_perm(qv, 0, 0x4140) * (uint32_t)sc + add;
                            const uint32_t pb = __byte_perm(qv, 0, 0x4342) * (uint32_t)sc + add;
                            v[i] = __byte_perm(pa, pb, 0x6420) ^ 0x80808080u;
                            v[8 + i] = __byte_perm(pa, pb, 0x7531) ^ 0x80808080u;
                        }
                        tmem_st16(tmem + lane_off + TM_A + 16 * ks, v);
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sh.a_full[ks]);
                    }
                }
                mbar_arrive(&sh.w_empty[ws]);
                if (++ws == C::W_STAGES) { ws = 0; wph ^= 1; }
            }
        }
    unpack_done:;
    } else if (warp >= 8) {
        // ============================================================ epilogue
        const int quad = warp & 3;
        const int half = (warp - 8) >> 2;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        constexpr int HC = NTOK / 2;  // columns per epilogue warp
        // preset every accumulator column this warp owns
        {
            uint32_t cv[8];
#pragma unroll
            for (int i = 0; i < 8; i++) cv[i] = MAGIC_BITS;
            for (int r = 0; r < ACC_SETS; r++)
                for (int a = 0; a < C::NACC; a++)
                    for (int c = 0; c < HC; c += 8)
                        tmem_st8(tmem + lane_off + TM_ACC + (r * C::NACC + a) * NTOK + half * HC + c, cv);
            tmem_wait_st();
            tc_fence_before();
            for (int r = 0; r < ACC_SETS; r++) mbar_arrive(&sh.acc_empty[r]);
        }
        uint32_t bs = 0, bph = 0, r = 0, rph = 0, ss = 0, sph = 0;
        for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
            const Unit un = unit_of(args, u);
            const int T = (un.len + NTOK - 1) / NTOK;
            const Segment& sg = args.seg[un.seg];
            float acc[TMAX][HC];
#pragma unroll
            for (int t = 0; t < TMAX; t++)
#pragma unroll
                for (int j = 0; j < HC; j++) acc[t][j] = 0.0f;
            for (int s = 0; s < nsb; s++) {
                if (!wait_bar_warp(sh, &sh.s_full[ss], sph)) goto epi_done;
                const float2 dd = sh.dd[ss][row];
                mbar_arrive(&sh.s_empty[ss]);
                if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
#pragma unroll
                for (int tt = 0; tt < TMAX; tt++) {
                    if (tt < T) {
                        const int ntok = min(NTOK, un.len - tt * NTOK);
                        if (!wait_bar_warp(sh, &sh.acc_full[r], rph)) goto epi_done;
                        if (!wait_bar_warp(sh, &sh.b_full[bs], bph)) goto epi_done;
                        tc_fence_after();
                        const uint32_t acc_t = tmem + lane_off + TM_ACC + r * C::NACC * NTOK + half * HC;
                        const float* da = reinterpret_cast<const float*>(b_stage + bs * C::B_STAGE + C::B_Q + C::B_SUMS);
#pragma unroll
                        for (int c = 0; c < HC; c += 8) {
                            if (half * HC + c < ntok) {
                                uint32_t x0[8], x1[8], x2[8], x3[8];
                                tmem_ld8(acc_t + c, x0);
                                tmem_ld8(acc_t + NTOK + c, x1);
                                if constexpr (QT == 12) {
                                    tmem_ld8(acc_t + 2 * NTOK + c, x2);
                                    tmem_ld8(acc_t + 3 * NTOK + c, x3);
                                }
                                tmem_wait_ld();
                                uint32_t cv[8];
#pragma unroll
                                for (int i = 0; i < 8; i++) cv[i] = MAGIC_BITS;
                                tmem_st8(acc_t + c, cv);
                                tmem_st8(acc_t + NTOK + c, cv);
                                if constexpr (QT == 12) {
                                    tmem_st8(acc_t + 2 * NTOK + c, cv);
                                    tmem_st8(acc_t + 3 * NTOK + c, cv);
                                }
                                if constexpr (DBG) {
#pragma unroll
                                    for (int i = 0; i < 8; i++) {
                                        const int64_t m = un.m0 + tt * NTOK + half * HC + c + i;
                                        if (m < args.m_out) {
                                            const int n = (int)(un.tile * TROWS + row);
                                            const int64_t o = (m * args.dbg_N + n) * nsb + s;
                                            if (QT == 12) {
                                                args.dbg_S[o] = (int32_t)(x0[i] - MAGIC_BITS) + 8 * (int32_t)(x1[i] - MAGIC_BITS);
                                                args.dbg_Smin[o] = (int32_t)(x2[i] - MAGIC_BITS) + 256 * (int32_t)(x3[i] - MAGIC_BITS);
                                            } else {
                                                args.dbg_S[o] = (int32_t)(x0[i] - MAGIC_BITS) + 256 * (int32_t)(x1[i] - MAGIC_BITS);
                                            }
                                        }
                                    }
                                } else {
                                    const float4 da0 = *reinterpret_cast<const float4*>(da + half * HC + c);
                                    const float4 da1 = *reinterpret_cast<const float4*>(da + half * HC + c + 4);
                                    const float dav[8] = {da0.x, da0.y, da0.z, da0.w, da1.x, da1.y, da1.z, da1.w};
#pragma unroll
                                    for (int i = 0; i < 8; i++) {
                                        float t;
                                        if constexpr (QT == 12) {
                                            const float S = fmaf(__uint_as_float(x1[i]), 8.0f, -9.0f * MAGIC) + __uint_as_float(x0[i]);
                                            const float Sm = fmaf(__uint_as_float(x3[i]), 256.0f, -257.0f * MAGIC) + __uint_as_float(x2[i]);
                                            t = fmaf(Sm, dd.y, S * dd.x);
                                        } else {
                                            const float S = fmaf(__uint_as_float(x1[i]), 256.0f, -257.0f * MAGIC) + __uint_as_float(x0[i]);
                                            t = S * dd.x;
                                        }
                                        acc[tt][c + i] = fmaf(t, dav[i], acc[tt][c + i]);
                                    }
                                }
                            }
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sh.acc_empty[r]);
                        mbar_arrive(&sh.b_empty[bs]);
                        if (++bs == C::B_STAGES) { bs = 0; bph ^= 1; }
                        if (++r == ACC_SETS) { r = 0; rph ^= 1; }
                    }
                }
            }
            if constexpr (!DBG) {
                float* out = sg.out;
                const int64_t n = un.tile * TROWS + row;
#pragma unroll
                for (int tt = 0; tt < TMAX; tt++) {
                    if (tt < T) {
#pragma unroll
                        for (int j = 0; j < HC; j++) {
                            const int64_t m = un.m0 + tt * NTOK + half * HC + j;
                            if (m < args.m_out && m < un.m0 + un.len) out[m * sg.ldo + n] = acc[tt][j];
                        }
                    }
                }
            }
        }
    epi_done:;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

template <int QT>
constexpr size_t gemm_smem_bytes() {
    using C = GemmCfg<QT>;
    return (size_t)C::W_STAGES * C::TILE + (size_t)C::B_STAGES * C::B_STAGE + sizeof(GemmShared);
}

}  // namespace dllm
