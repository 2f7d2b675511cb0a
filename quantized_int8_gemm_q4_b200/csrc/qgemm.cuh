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
// The d-term, on the int8 tensor pipe, exactly.  The tensor core multiplies 8-bit
// operands, and q*sc needs 10 bits (Q4_K) or 13 bits (Q6_K), so the weight operand
// is split into two 8-bit planes whose integer results are recombined exactly:
//   Q4_K: sc = lo3 + 8*hi3 (3 bits each); plane 0 = q*lo3, plane 1 = q*hi3, both in
//         0..105 (u8).  S = P0 + 8*P1.
//   Q6_K: v = (q-32)*sc + 32896 lies in [28800, 36992]; plane 0 = (v & 255) - 128,
//         plane 1 = (v >> 8) - 128 (both s8), and plane0 + 256*plane1 = (q-32)*sc.
// Each plane accumulator stays within 2^22 in magnitude.  The first MMA of each
// super-block overwrites it, and the epilogue adds the bit pattern of 1.5*2^23 to
// the int32 it reads, which makes an f32 equal to exactly 1.5*2^23 + value; S then
// takes one FFMA and one FADD (packed f32x2), with no integer-to-float instruction.
// The epilogue then accumulates da * d * S in f32 registers.
//
// The min term (Q4_K), on the tf32 tensor pipe.  Its per-super-block factor
// dmin[n] * da[m] is a product of a row term and a column term, so
//   -sum_sb da dmin Smin = sum over (sb, j) of (-dmin m_j)[n] * (da sum32_j)[m],
// a GEMM with one K step per sub-block.  Both operands are split as hi + lo with hi
// exact in tf32 (-dmin m_j is exact in hi + lo; da*sum32_j loses at most 2^-22 of
// itself), and hi*hi + hi*lo + lo*hi accumulate in an f32 tensor-memory accumulator
// over the whole K range, read once per work unit.  Its error is below 2^-21 of the
// min term's magnitude, inside the 1e-6 * sum|terms| tolerance.
//
// Roles (16 warps, one CTA per SM, persistent over work units):
//   warp 0      producer: bulk copies of weight tiles and activation tiles into
//               shared-memory rings
//   warps 1-2   MMA issue (warp 1 also allocates tensor memory).  One thread can
//               issue a tcgen05.mma only every ~28 ns, longer than a 64-token MMA
//               takes, so the two token tiles of a super-block go to two warps, each
//               with its own accumulator set and a short wait/issue/commit loop
//   warp 3      idle
//   warps 4-7   unpack: thread = weight row; decode the super-block, build the two
//               weight planes per K-step of 32 into a tensor-memory ring of half
//               super-blocks (the A operand), the min-term A operand into shared
//               memory, and the f32 d; a half is published only once the
//               super-block's activation stages have landed
//   warps 8-15  epilogue: two warps per tensor-memory lane quadrant, each on half of
//               the token columns; per super-block, read the two plane accumulators,
//               release them to the issuer, and accumulate the f32 result in registers
//
// A work unit is (128 weight rows, up to 128 canvas rows, one K-chunk).  The number
// of K-chunks per tile depends only on N, K and the SM count, never on M or on the
// rows requested, and chunk partials are summed in chunk order by whichever CTA
// finishes a tile last; so results are deterministic and the same for every M.
#pragma once
#include "layout.cuh"

namespace dllm {

constexpr uint32_t MAGIC_BITS = 0x4B400000u;  // 1.5 * 2^23
constexpr float MAGIC = 12582912.0f;
constexpr int GEMM_THREADS = 512;
constexpr int UNIT_TOKENS = 128;
constexpr int NTOK = 64;                           // token columns per MMA and per accumulator
constexpr int TMAX = UNIT_TOKENS / NTOK;           // token tiles per unit
constexpr int HC = NTOK / 2;                       // token columns per epilogue warp
constexpr int MAX_KC = 16;                         // K-chunks per tile, at most
constexpr int ISSUERS = 2;                         // MMA-issuing warps
constexpr int S_SLOTS = 4;                         // d ring (unpack -> epilogue)
constexpr int ACC_SETS = 2;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s

// tensor-memory columns
// tensor-memory columns: the A ring (RING halves of a super-block, each 4 K-step slots
// of 16 columns: plane 0 | plane 1), then ACC_SETS x 2 planes x NTOK accumulator
// columns, then (Q4_K) TMAX x NTOK f32 min-term accumulator columns
constexpr uint32_t TM_A = 0;
constexpr uint32_t TM_COLS = 512;

// Activation "sums" operand of one super-block: per 8-row group 512 bytes =
// [hi j0-3 | hi j4-7 | lo j0-3 | lo j4-7] x [8 rows x 16 bytes].
constexpr int SUMS_GROUP = 512;

template <int QT>
struct GemmCfg;
template <>
struct GemmCfg<12> {  // Q4_K
    static constexpr int TILE = Q4K_TILE;
    static constexpr bool MIN = true;
    static constexpr int W_STAGES = 4;
    static constexpr int B_STAGES = 4;
    static constexpr int B_Q = NTOK * 256;
    static constexpr int B_SUMS = NTOK / 8 * SUMS_GROUP;
    static constexpr int B_STAGE = B_Q + B_SUMS + NTOK * 4;
    static constexpr int MINA = 2 * 4096;  // -dmin*m_j as [hi | lo], canonical K-major 128 rows x 32 B
    static constexpr int RING = 2;         // A ring: one super-block (the min accumulators take the rest)
    static constexpr uint32_t TM_ACC = 64 * RING;
    static constexpr uint32_t TM_MIN = TM_ACC + ACC_SETS * 2 * NTOK;
};
template <>
struct GemmCfg<14> {  // Q6_K
    static constexpr int TILE = Q6K_TILE;
    static constexpr bool MIN = false;
    static constexpr int W_STAGES = 3;
    static constexpr int B_STAGES = 4;
    static constexpr int B_Q = NTOK * 256;
    static constexpr int B_SUMS = 0;
    static constexpr int B_STAGE = B_Q + B_SUMS + NTOK * 4;
    static constexpr int MINA = 0;
    static constexpr int RING = 4;  // A ring: two super-blocks, so the unpack runs one ahead
    static constexpr uint32_t TM_ACC = 64 * RING;
    static constexpr uint32_t TM_MIN = 0;
};

struct Segment {
    const uint8_t* w;  // repacked weights
    float* out;
    int64_t ldo;
    int32_t tile0;     // first global n-tile of this segment
};

struct GemmArgs {
    Segment seg[3];
    int nseg;
    int32_t n_tiles;   // total 128-row tiles over all segments
    int32_t nsb;       // K / 256
    int32_t kc;        // K-chunks per tile (uniform split: tail_k == 0)
    // Tail split (tail_k > 0): tiles [0, full_tiles) run whole, one round of one tile per
    // CTA at a time; each remaining tile is cut into K-pieces so that the pieces fill
    // exactly one more unit per CTA: the first tail_big of them into tail_k + 1 pieces,
    // the others into tail_k.
    int32_t full_tiles, tail_k, tail_big;
    int64_t n_units;   // work units of the launch (token super-tiles included)
    const int8_t* q;   // tiled activations
    const float* scale;
    const uint8_t* sums;
    int64_t Mp;        // rows of the activation layout (multiple of 16)
    int64_t m_out;     // output rows
    int32_t n_st;      // token super-tiles
    int32_t mu;        // tokens per super-tile (multiple of 16)
    uint32_t* counters;  // [n_tiles * n_st], when kc > 1
    float* partials;     // [units][mu/4][128 rows][4 tokens], when kc > 1
    int32_t* dbg_S;    // debug: per-super-block integer S instead of f32 (nullable)
    int32_t stall;     // test: the producer issues nothing, so every other role's wait runs out
    int64_t dbg_N;
};

struct GemmShared {
    uint64_t w_full[8], w_empty[8];
    uint64_t b_full[8], b_empty[8];
    uint64_t a_full[4], a_empty[4];  // A ring slots: super-block halves (K-steps 0-3, 4-7 + the min-term A)
    uint64_t s_full[S_SLOTS], s_empty[S_SLOTS];
    uint64_t acc_full[ACC_SETS], acc_empty[ACC_SETS];
    uint64_t min_empty;
    uint64_t final_bar[4];
    uint64_t epi_bar;
    uint32_t tmem_base;
    volatile int abort_flag;
    int last_flag;
    float dd[S_SLOTS][TROWS];
};

// Bounded wait on an mbarrier phase; false if this CTA is aborting.  Waiting threads
// sleep inside try_wait.  Raises the abort flag and the device error word when the
// limit runs out.
__device__ __forceinline__ bool wait_bar(GemmShared& sh, uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
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
// Bounded barrier among the 256 epilogue threads.
__device__ __forceinline__ bool epi_sync(GemmShared& sh, uint32_t& phase) {
    mbar_arrive(&sh.epi_bar);
    const bool ok = wait_bar_warp(sh, &sh.epi_bar, phase);
    phase ^= 1;
    return ok;
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
// This warp's HC = 32 consecutive accumulator columns.
__device__ __forceinline__ void load_cols(uint32_t taddr, uint32_t (&x)[HC]) {
    tmem_ld16(taddr, x);
    tmem_ld16(taddr + 16, x + 16);
}

struct Unit {
    int seg;
    int64_t tile;   // tile index inside the segment
    int32_t gtile;  // global tile index
    int32_t st;     // token super-tile
    int32_t chunk;  // K-piece of the tile
    int64_t m0;     // first token of the super-tile
    int32_t len;    // tokens in the super-tile (multiple of 16)
    int32_t sb0, sb1;
    int32_t np;        // K-pieces of the tile (1: the unit writes the output itself)
    int64_t slot0;     // partial-sum slot of the tile's piece 0 (same super-tile)
    int32_t pstride;   // slot distance between consecutive pieces
};

template <bool TAIL>
__device__ __forceinline__ Unit unit_of(const GemmArgs& a, int64_t u) {
    Unit r;
    if constexpr (!TAIL) {
        r.chunk = (int32_t)(u % a.kc);
        const int64_t ts = u / a.kc;
        r.st = (int32_t)(ts % a.n_st);
        r.gtile = (int32_t)(ts / a.n_st);
        r.sb0 = (int32_t)((int64_t)r.chunk * a.nsb / a.kc);
        r.sb1 = (int32_t)((int64_t)(r.chunk + 1) * a.nsb / a.kc);
        r.np = a.kc;
        r.slot0 = u - r.chunk;  // partial slots are unit indices
        r.pstride = 1;
    } else {
        // unit u = (tile piece cu, super-tile st), st fastest; partial slots count the
        // tail units only.  32-bit arithmetic: the host keeps n_units below 2^31 here.
        const uint32_t uu = (uint32_t)u, nst = (uint32_t)a.n_st;
        const uint32_t cu = uu / nst;
        r.st = (int32_t)(uu - cu * nst);
        if (cu < (uint32_t)a.full_tiles) {
            r.gtile = (int32_t)cu;
            r.chunk = 0;
            r.np = 1;
        } else {
            const uint32_t i = cu - (uint32_t)a.full_tiles;
            const uint32_t big = (uint32_t)a.tail_big * (uint32_t)(a.tail_k + 1);
            const uint32_t np = i < big ? (uint32_t)a.tail_k + 1 : (uint32_t)a.tail_k;
            const uint32_t i2 = i < big ? i : i - big;
            const uint32_t j = i2 / np;
            r.np = (int32_t)np;
            r.chunk = (int32_t)(i2 - j * np);
            r.gtile = a.full_tiles + (int32_t)(i < big ? j : (uint32_t)a.tail_big + j);
        }
        r.sb0 = (int32_t)((uint32_t)r.chunk * (uint32_t)a.nsb / (uint32_t)r.np);
        r.sb1 = (int32_t)((uint32_t)(r.chunk + 1) * (uint32_t)a.nsb / (uint32_t)r.np);
        r.slot0 = (int64_t)((cu - (uint32_t)r.chunk - (uint32_t)a.full_tiles) * nst + (uint32_t)r.st);
        r.pstride = a.n_st;
    }
    r.seg = 0;
    if (a.nseg > 1 && r.gtile >= a.seg[1].tile0) r.seg = 1;
    if (a.nseg > 2 && r.gtile >= a.seg[2].tile0) r.seg = 2;
    r.tile = r.gtile - a.seg[r.seg].tile0;
    r.m0 = (int64_t)r.st * a.mu;
    r.len = (int32_t)min((int64_t)a.mu, a.Mp - r.m0);
    return r;
}

template <int QT>
constexpr bool tmem_fits() {
    using C = GemmCfg<QT>;
    return C::TM_ACC + ACC_SETS * 2 * NTOK + (C::MIN ? TMAX * NTOK : 0) <= TM_COLS &&
           (!C::MIN || C::TM_MIN == C::TM_ACC + ACC_SETS * 2 * NTOK) && C::RING <= 4 && C::RING % 2 == 0;
}
static_assert(tmem_fits<12>() && tmem_fits<14>(), "tensor-memory columns over budget");

template <int QT, bool DBG, bool TAIL>
__global__ void __launch_bounds__(GEMM_THREADS, 1) qgemm_kernel(const __grid_constant__ GemmArgs args) {
    using C = GemmCfg<QT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* w_stage = smem_raw;
    uint8_t* b_stage = w_stage + C::W_STAGES * C::TILE;
    uint8_t* mina = b_stage + C::B_STAGES * C::B_STAGE;
    GemmShared& sh = *reinterpret_cast<GemmShared*>(mina + C::MINA);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_units = args.n_units;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::W_STAGES; i++) { mbar_init(&sh.w_full[i], 1); mbar_init(&sh.w_empty[i], 128); }
        for (int i = 0; i < C::B_STAGES; i++) { mbar_init(&sh.b_full[i], 1); mbar_init(&sh.b_empty[i], 256); }
        for (int i = 0; i < C::RING; i++) { mbar_init(&sh.a_full[i], 128); mbar_init(&sh.a_empty[i], ISSUERS); }
        for (int i = 0; i < S_SLOTS; i++) { mbar_init(&sh.s_full[i], 128); mbar_init(&sh.s_empty[i], 256); }
        for (int i = 0; i < ACC_SETS; i++) { mbar_init(&sh.acc_full[i], 1); mbar_init(&sh.acc_empty[i], 256); }
        mbar_init(&sh.min_empty, 256);
        for (int i = 0; i < 4; i++) mbar_init(&sh.final_bar[i], 1);
        mbar_init(&sh.epi_bar, 256);
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
    // Everything above, and the producer's L2 prefetch of its first weight tiles, may
    // overlap the previous kernel on the stream; every access to global memory that
    // earlier work can write comes after pdl_wait in the role that makes it.
    if (threadIdx.x == 0) pdl_trigger();

    if (warp < 4) {
        setmaxnreg_dec<48>();
        if (warp == 0) {
            // ======================================================== producer
            uint32_t ws = 0, wph = 0, bs = 0, bph = 0;
            // stages with a copy issued (bit i) and the phase it completes (bit i)
            uint32_t w_iss = 0, w_php = 0, b_iss = 0, b_php = 0;
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            const int64_t n_prod = args.stall ? 0 : n_units;
            if (lane == 0 && blockIdx.x < n_prod) {
                const Unit un = unit_of<TAIL>(args, blockIdx.x);
                const uint8_t* wt = args.seg[un.seg].w + (size_t)un.tile * args.nsb * C::TILE;
                for (int s = un.sb0; s < un.sb1 && s < un.sb0 + C::W_STAGES; s++)
                    prefetch_l2(wt + (size_t)s * C::TILE, C::TILE);
            }
            pdl_wait();
            for (int64_t u = blockIdx.x; u < n_prod; u += gridDim.x) {
                const Unit un = unit_of<TAIL>(args, u);
                const uint8_t* wt = args.seg[un.seg].w + (size_t)un.tile * args.nsb * C::TILE;
                const int T = (un.len + NTOK - 1) / NTOK;
                for (int s = un.sb0; s < un.sb1; s++) {
                    if (!wait_bar_warp(sh, &sh.w_empty[ws], wph ^ 1)) goto prod_done;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&sh.w_full[ws], C::TILE);
                        bulk_g2s_hint(w_stage + ws * C::TILE, wt + (size_t)s * C::TILE, C::TILE, &sh.w_full[ws],
                                      pol_w);
                    }
                    w_iss |= 1u << ws;
                    w_php = (w_php & ~(1u << ws)) | (wph << ws);
                    if (++ws == C::W_STAGES) { ws = 0; wph ^= 1; }
                    for (int tt = 0; tt < T; tt++) {
                        const int64_t t0 = un.m0 + (int64_t)tt * NTOK;
                        const int ntok = min(NTOK, un.len - tt * NTOK);
                        if (!wait_bar_warp(sh, &sh.b_empty[bs], bph ^ 1)) goto prod_done;
                        if (lane == 0) {
                            uint8_t* st = b_stage + bs * C::B_STAGE;
                            const uint32_t sums_bytes = C::B_SUMS ? ntok / 8 * SUMS_GROUP : 0;
                            mbar_arrive_expect_tx(&sh.b_full[bs], ntok * 256 + sums_bytes + ntok * 4);
                            bulk_g2s_hint(st, args.q + ((size_t)s * args.Mp + t0) * 256, ntok * 256, &sh.b_full[bs],
                                          pol_a);
                            if (C::B_SUMS)
                                bulk_g2s_hint(st + C::B_Q, args.sums + ((size_t)s * args.Mp + t0) / 8 * SUMS_GROUP,
                                              sums_bytes, &sh.b_full[bs], pol_a);
                            bulk_g2s_hint(st + C::B_Q + C::B_SUMS, args.scale + (size_t)s * args.Mp + t0, ntok * 4,
                                          &sh.b_full[bs], pol_a);
                        }
                        b_iss |= 1u << bs;
                        b_php = (b_php & ~(1u << bs)) | (bph << bs);
                        if (++bs == C::B_STAGES) { bs = 0; bph ^= 1; }
                    }
                }
            }
        prod_done:
            if (sh.abort_flag) {  // never leave with bulk copies in flight into this CTA's shared memory
                for (int i = 0; i < C::W_STAGES; i++)
                    if ((w_iss >> i) & 1u) (void)wait_bar(sh, &sh.w_full[i], (w_php >> i) & 1u);
                for (int i = 0; i < C::B_STAGES; i++)
                    if ((b_iss >> i) & 1u) (void)wait_bar(sh, &sh.b_full[i], (b_php >> i) & 1u);
            }
        } else {
            // ======================================================== MMA issuers
            // The (super-block, token tile) items of this CTA alternate between warps 1
            // and 2, and item i owns accumulator set i % 2; with two token tiles each
            // issuer owns one tile.  Per super-block an issuer waits for each half of
            // the A ring, issues its item's MMAs on that half (both planes; the min
            // term with the second half), and commits once to the half's release
            // barrier, so every release takes one arrival from each issuer.  Warp 3
            // issues nothing.
            const int who = warp - 1;
            const bool leader = lane == 0;
            if (who < ISSUERS) {
                uint32_t item = 0, sbc = 0, uc = 0;
                for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, uc++) {
                    const Unit un = unit_of<TAIL>(args, u);
                    const int T = (un.len + NTOK - 1) / NTOK;
                    for (int s = un.sb0; s < un.sb1; s++, sbc++, item += T) {
#pragma unroll 1
                        for (int half = 0; half < 2; half++) {
                            const uint32_t hc = 2 * sbc + half, slot = hc % C::RING;
                            if (!wait_bar_warp(sh, &sh.a_full[slot], (hc / C::RING) & 1)) goto mma_done;
                            for (int tt = 0; tt < T; tt++) {
                                const uint32_t it = item + tt;
                                if ((int)(it & 1) != who) continue;
                                const uint32_t set = it & 1;
                                const uint32_t bst = it % C::B_STAGES;
                                const int ntok = min(NTOK, un.len - tt * NTOK);
                                if (half == 0) {
                                    // (the item's activation stage is full: the unpack waited for it
                                    // before publishing the A-ring half waited on above)
                                    if (!wait_bar_warp(sh, &sh.acc_empty[set], (it >> 1) & 1)) goto mma_done;
                                } else if (C::MIN && s == un.sb0) {
                                    // a unit's first min-term MMAs overwrite the min accumulators:
                                    // the previous unit's epilogue must have read them out
                                    if (!wait_bar_warp(sh, &sh.min_empty, (uc & 1) ^ 1)) goto mma_done;
                                }
                                tc_fence_after();
                                if (leader) {
                                    const uint32_t st = smem_u32(b_stage + bst * C::B_STAGE);
                                    const uint32_t id = QT == 12 ? idesc_i8(128, ntok, 0, 1) : idesc_i8(128, ntok, 1, 1);
                                    const uint32_t d0 = tmem + C::TM_ACC + set * 2 * NTOK;
                                    const uint32_t a0 = tmem + TM_A + 64 * slot;
                                    const uint64_t b0 = sdesc_kmajor_noswz(st, 128, 2048) + 64 * half;
#pragma unroll
                                    for (int ks = 0; ks < 4; ks++) mma_i8_ts(d0, a0 + 16 * ks, b0 + 16 * ks, id, half | ks ? 1u : 0u);
#pragma unroll
                                    for (int ks = 0; ks < 4; ks++) mma_i8_ts(d0 + NTOK, a0 + 16 * ks + 8, b0 + 16 * ks, id, half | ks ? 1u : 0u);
                                    if (C::MIN && half == 1) {
                                        const uint32_t d = tmem + C::TM_MIN + tt * NTOK;
                                        const uint32_t idm = idesc_tf32(128, ntok);
                                        const uint32_t ma = smem_u32(mina);
                                        const uint64_t a_hi = sdesc_kmajor_noswz(ma, 128, 256);
                                        const uint64_t a_lo = sdesc_kmajor_noswz(ma + 4096, 128, 256);
                                        const uint64_t b_hi = sdesc_kmajor_noswz(st + C::B_Q, 128, SUMS_GROUP);
                                        const uint64_t b_lo = sdesc_kmajor_noswz(st + C::B_Q + 256, 128, SUMS_GROUP);
                                        mma_tf32_ss(d, a_hi, b_hi, idm, s > un.sb0 ? 1u : 0u);
                                        mma_tf32_ss(d, a_hi, b_lo, idm, 1);
                                        mma_tf32_ss(d, a_lo, b_hi, idm, 1);
                                    }
                                    if (half == 1) tc_commit(&sh.acc_full[set]);
                                }
                                __syncwarp();
                            }
                            if (leader) tc_commit(&sh.a_empty[slot]);
                            __syncwarp();
                        }
                    }
                }
            }
        mma_done:
            // every MMA this warp issued has completed before tensor memory is freed
            if (leader) tc_commit(&sh.final_bar[who]);
            __syncwarp();
            (void)wait_bar_warp(sh, &sh.final_bar[who], 0);
        }
    } else if (warp < 8) {
        setmaxnreg_dec<80>();
        // ============================================================ unpack
        // Per super-block: decode this row, then build the planes of K-steps 0-3 and
        // publish them together, then K-steps 4-7 (and the min-term A), so the MMAs of
        // a super-block can start while the second half is still being built.
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        uint32_t ws = 0, wph = 0, ss = 0, sph = 0, sbc = 0, itm = 0;
        for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
            const Unit un = unit_of<TAIL>(args, u);
            const int T = (un.len + NTOK - 1) / NTOK;
            for (int s = un.sb0; s < un.sb1; s++, sbc++, itm += T) {
                if (!wait_bar_warp(sh, &sh.w_full[ws], wph)) goto unpack_done;
                // the super-block's activation stages (one per token tile) are full before
                // any half of its A ring is published, so the MMA issuer need not wait on them
                for (int tt = 0; tt < T; tt++) {
                    const uint32_t it = itm + tt;
                    if (!wait_bar_warp(sh, &sh.b_full[it % C::B_STAGES], (it / C::B_STAGES) & 1)) goto unpack_done;
                }
                const uint8_t* tl = w_stage + ws * C::TILE;
                if constexpr (QT == 12) {
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_SC + 12 * row);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_SC + 12 * row + 4);
                    const uint32_t b2 = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_SC + 12 * row + 8);
                    const uint32_t dm = *reinterpret_cast<const uint32_t*>(tl + Q4K_OFF_D + 4 * row);
                    uint32_t sc[8];
                    float nmin[8];  // -dmin * m_j, exact in f32
                    const float d = __half2float(__ushort_as_half((unsigned short)(dm & 0xFFFF)));
                    const float dmin = __half2float(__ushort_as_half((unsigned short)(dm >> 16)));
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        sc[j] = (b0 >> (8 * j)) & 63;
                        sc[j + 4] = ((b2 >> (8 * j)) & 15) | (((b0 >> (8 * j + 6)) & 3) << 4);
                        const uint32_t m_lo = (b1 >> (8 * j)) & 63;
                        const uint32_t m_hi = ((b2 >> (8 * j + 4)) & 15) | (((b1 >> (8 * j + 6)) & 3) << 4);
                        nmin[j] = -dmin * (float)m_lo;
                        nmin[j + 4] = -dmin * (float)m_hi;
                    }
                    if (!wait_bar_warp(sh, &sh.s_empty[ss], sph ^ 1)) goto unpack_done;
                    sh.dd[ss][row] = d;
                    mbar_arrive(&sh.s_full[ss]);
                    if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
#pragma unroll
                    for (int half = 0; half < 2; half++) {
                        const uint32_t hc = 2 * sbc + half, slot = hc % C::RING;
                        if (!wait_bar_warp(sh, &sh.a_empty[slot], ((hc / C::RING) & 1) ^ 1)) goto unpack_done;
                        if (half == 1) {
                            // -dmin*m_j as tf32 hi + lo: row `row` of the canonical K-major
                            // layout (8-row groups of 256 bytes, two 16-byte K chunks)
                            float hi[8], lo[8];
#pragma unroll
                            for (int j = 0; j < 8; j++) split_tf32(nmin[j], hi[j], lo[j]);
                            uint8_t* base = mina + (row >> 3) * 256 + (row & 7) * 16;
                            *reinterpret_cast<float4*>(base) = make_float4(hi[0], hi[1], hi[2], hi[3]);
                            *reinterpret_cast<float4*>(base + 128) = make_float4(hi[4], hi[5], hi[6], hi[7]);
                            *reinterpret_cast<float4*>(base + 4096) = make_float4(lo[0], lo[1], lo[2], lo[3]);
                            *reinterpret_cast<float4*>(base + 4096 + 128) = make_float4(lo[4], lo[5], lo[6], lo[7]);
                            fence_proxy_async_smem();
                        }
#pragma unroll
                        for (int cc = 0; cc < 2; cc++) {
                            const int c = 2 * half + cc;  // 32-byte quant chunk: sub-blocks 2c, 2c+1
                            const uint4 p0 = *reinterpret_cast<const uint4*>(tl + ((2 * c) * TROWS + row) * 16);
                            const uint4 p1 = *reinterpret_cast<const uint4*>(tl + ((2 * c + 1) * TROWS + row) * 16);
                            const uint32_t wv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                            for (int h = 0; h < 2; h++) {
                                const int ks = 2 * c + h;
                                const uint32_t lo3 = sc[ks] & 7, hi3 = sc[ks] >> 3;
                                uint32_t v[16];
#pragma unroll
                                for (int i = 0; i < 8; i++) {
                                    const uint32_t nib = (wv[i] >> (4 * h)) & 0x0F0F0F0Fu;
                                    v[i] = nib * lo3;
                                    v[8 + i] = nib * hi3;
                                }
                                tmem_st16(tmem + lane_off + TM_A + 64 * slot + 16 * (ks & 3), v);
                            }
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sh.a_full[slot]);
                    }
                } else {
                    const uint4 scv = *reinterpret_cast<const uint4*>(tl + Q6K_OFF_SC + 16 * row);
                    const uint32_t scw[4] = {scv.x, scv.y, scv.z, scv.w};
                    const float d = __half2float(
                        __ushort_as_half(*reinterpret_cast<const unsigned short*>(tl + Q6K_OFF_D + 2 * row)));
                    if (!wait_bar_warp(sh, &sh.s_empty[ss], sph ^ 1)) goto unpack_done;
                    sh.dd[ss][row] = d;
                    mbar_arrive(&sh.s_full[ss]);
                    if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
#pragma unroll
                    for (int half = 0; half < 2; half++) {
                        const uint32_t hc = 2 * sbc + half, slot = hc % C::RING;
                        if (!wait_bar_warp(sh, &sh.a_empty[slot], ((hc / C::RING) & 1) ^ 1)) goto unpack_done;
#pragma unroll
                        for (int kq = 0; kq < 4; kq++) {
                            const int ks = 4 * half + kq;
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
                            uint32_t v[16];
#pragma unroll
                            for (int i = 0; i < 8; i++) {
                                const uint32_t qv =
                                    ((lw[i] >> sh_lo) & 0x0F0F0F0Fu) | (((hw[i] >> sh_hi) & 0x03030303u) << 4);
                                const int32_t scs = i < 4 ? sca : scb;
                                const uint32_t add = i < 4 ? adda : addb;
                                const uint32_t pa = __byte_perm(qv, 0, 0x4140) * (uint32_t)scs + add;
                                const uint32_t pb = __byte_perm(qv, 0, 0x4342) * (uint32_t)scs + add;
                                v[i] = __byte_perm(pa, pb, 0x6420) ^ 0x80808080u;
                                v[8 + i] = __byte_perm(pa, pb, 0x7531) ^ 0x80808080u;
                            }
                            tmem_st16(tmem + lane_off + TM_A + 64 * slot + 16 * (ks & 3), v);
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sh.a_full[slot]);
                    }
                }
                mbar_arrive(&sh.w_empty[ws]);
                if (++ws == C::W_STAGES) { ws = 0; wph ^= 1; }
            }
        }
    unpack_done:;
    } else {
        setmaxnreg_inc<192>();
        // ============================================================ epilogue
        pdl_wait();  // outputs, partials and counters may be in use by earlier work
        const int quad = warp & 3;
        const int half = (warp - 8) >> 2;
        const int row = quad * 32 + lane;
        const int etid = threadIdx.x - 256;  // 0..255
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        for (int r = 0; r < ACC_SETS; r++) mbar_arrive(&sh.acc_empty[r]);
        const float2 k8 = make_float2(8.0f, 8.0f), k256 = make_float2(256.0f, 256.0f);
        const float2 m9 = make_float2(-9.0f * MAGIC, -9.0f * MAGIC);
        const float2 m257 = make_float2(-257.0f * MAGIC, -257.0f * MAGIC);
        uint32_t bs = 0, bph = 0, r = 0, rph = 0, ss = 0, sph = 0, epi_ph = 0;
        for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
            const Unit un = unit_of<TAIL>(args, u);
            const int T = (un.len + NTOK - 1) / NTOK;
            const Segment& sg = args.seg[un.seg];
            float2 acc[TMAX][HC / 2];
#pragma unroll
            for (int t = 0; t < TMAX; t++)
#pragma unroll
                for (int j = 0; j < HC / 2; j++) acc[t][j] = make_float2(0.0f, 0.0f);
            for (int s = un.sb0; s < un.sb1; s++) {
                if (!wait_bar_warp(sh, &sh.s_full[ss], sph)) goto epi_done;
                const float dv = sh.dd[ss][row];
                mbar_arrive(&sh.s_empty[ss]);
                if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
                const float2 d2 = make_float2(dv, dv);
#pragma unroll
                for (int tt = 0; tt < TMAX; tt++) {
                    if (tt < T) {
                        const int ntok = min(NTOK, un.len - tt * NTOK);
                        if (!wait_bar_warp(sh, &sh.acc_full[r], rph)) goto epi_done;
                        if (!wait_bar_warp(sh, &sh.b_full[bs], bph)) goto epi_done;
                        tc_fence_after();
                        const uint32_t acc_t = tmem + lane_off + C::TM_ACC + r * 2 * NTOK + half * HC;
                        const float* da = reinterpret_cast<const float*>(b_stage + bs * C::B_STAGE + C::B_Q + C::B_SUMS);
                        // read both plane accumulators and release them to the MMA issuer
                        // (the next super-block's first MMA overwrites them) before doing
                        // any arithmetic on the values
                        if (half * HC < ntok) {
                            uint32_t x0[HC], x1[HC];
                            load_cols(acc_t, x0);
                            load_cols(acc_t + NTOK, x1);
                            tmem_wait_ld();
                            tc_fence_before();
                            mbar_arrive(&sh.acc_empty[r]);
                            if constexpr (DBG) {
#pragma unroll
                                for (int i = 0; i < HC; i++) {
                                    const int64_t m = un.m0 + tt * NTOK + half * HC + i;
                                    if (half * HC + i < ntok && m < args.m_out) {
                                        const int64_t n = un.tile * TROWS + row;
                                        const int32_t P0 = (int32_t)x0[i], P1 = (int32_t)x1[i];
                                        args.dbg_S[(m * args.dbg_N + n) * args.nsb + s] = P0 + (QT == 12 ? 8 : 256) * P1;
                                    }
                                }
                            } else {
#pragma unroll
                                for (int i = 0; i < HC / 2; i++) {
                                    // |P| < 2^22: adding the bits of 1.5*2^23 gives the f32 1.5*2^23 + P
                                    const float2 X0 = make_float2(__uint_as_float(x0[2 * i] + MAGIC_BITS),
                                                                  __uint_as_float(x0[2 * i + 1] + MAGIC_BITS));
                                    const float2 X1 = make_float2(__uint_as_float(x1[2 * i] + MAGIC_BITS),
                                                                  __uint_as_float(x1[2 * i + 1] + MAGIC_BITS));
                                    const float2 S = QT == 12 ? __fadd2_rn(__ffma2_rn(X1, k8, m9), X0)
                                                              : __fadd2_rn(__ffma2_rn(X1, k256, m257), X0);
                                    const float2 dav = *reinterpret_cast<const float2*>(da + half * HC + 2 * i);
                                    acc[tt][i] = __ffma2_rn(__fmul2_rn(S, d2), dav, acc[tt][i]);
                                }
                            }
                        } else {
                            tc_fence_before();
                            mbar_arrive(&sh.acc_empty[r]);
                        }
                        mbar_arrive(&sh.b_empty[bs]);
                        if (++bs == C::B_STAGES) { bs = 0; bph ^= 1; }
                        if (++r == ACC_SETS) { r = 0; rph ^= 1; }
                    }
                }
            }
            if constexpr (C::MIN) {
                // the min-term accumulators: complete, since every tile's last MMAs were
                // covered by the accumulator barriers waited on above
#pragma unroll
                for (int tt = 0; tt < TMAX; tt++) {
                    if (tt < T && half * HC < un.len - tt * NTOK) {
                        uint32_t y[HC];
                        load_cols(tmem + lane_off + C::TM_MIN + tt * NTOK + half * HC, y);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < HC / 2; i++)
                            acc[tt][i] = __fadd2_rn(acc[tt][i], make_float2(__uint_as_float(y[2 * i]), __uint_as_float(y[2 * i + 1])));
                    }
                }
                tc_fence_before();
                mbar_arrive(&sh.min_empty);
            }
            if constexpr (!DBG) {
                const int64_t n = un.tile * TROWS + row;
                // uniform split: every tile has kc pieces and partial slots are unit indices
                const int np = TAIL ? un.np : args.kc;
                if (np == 1) {
                    float* out = sg.out;
#pragma unroll
                    for (int tt = 0; tt < TMAX; tt++) {
                        if (tt < T) {
#pragma unroll
                            for (int j = 0; j < HC; j++) {
                                const int64_t m = un.m0 + tt * NTOK + half * HC + j;
                                if (m < args.m_out && m < un.m0 + un.len)
                                    out[m * sg.ldo + n] = j & 1 ? acc[tt][j / 2].y : acc[tt][j / 2].x;
                            }
                        }
                    }
                } else {
                    // this K-chunk's partial: [unit][mu/4][128 rows][4 tokens], so a thread's
                    // 4 consecutive tokens are one 16-byte store and a warp's 32 rows 512
                    // contiguous bytes (token counts are multiples of 16)
                    const int64_t my_slot = TAIL ? un.slot0 + (int64_t)un.chunk * un.pstride : u;
                    float* part = args.partials + (size_t)my_slot * args.mu * TROWS + row * 4;
#pragma unroll
                    for (int tt = 0; tt < TMAX; tt++) {
#pragma unroll
                        for (int q4 = 0; q4 < HC / 4; q4++) {
                            const int ml = tt * NTOK + half * HC + 4 * q4;
                            if (tt < T && ml < un.len)
                                __stcg(reinterpret_cast<float4*>(part + (size_t)(ml / 4) * TROWS * 4),
                                       make_float4(acc[tt][2 * q4].x, acc[tt][2 * q4].y, acc[tt][2 * q4 + 1].x,
                                                   acc[tt][2 * q4 + 1].y));
                        }
                    }
                    __threadfence();
                    if (!epi_sync(sh, epi_ph)) goto epi_done;
                    if (etid == 0) {
                        uint32_t* ctr = args.counters + (size_t)un.gtile * args.n_st + un.st;
                        const uint32_t old = atomicAdd(ctr, 1u);
                        // counters advance by 16 per call and split tile: the last of the
                        // np arrivals tops the counter up to the next multiple of 16
                        const int last = (int)(old & 15u) == np - 1;
                        if (last) atomicAdd(ctr, (uint32_t)(16 - np));
                        __threadfence();
                        sh.last_flag = last;
                    }
                    if (!epi_sync(sh, epi_ph)) goto epi_done;
                    if (sh.last_flag) {
                        // sum the piece partials in piece order; each token tile's 8 loads of
                        // 16 bytes are issued before any is used
                        for (int c2 = 0; c2 < np; c2++) {
                            const int64_t slot = TAIL ? un.slot0 + (int64_t)c2 * un.pstride : u - un.chunk + c2;
                            const float* part = args.partials + (size_t)slot * args.mu * TROWS + row * 4;
#pragma unroll
                            for (int tt = 0; tt < TMAX; tt++) {
                                float4 pv[HC / 4];
#pragma unroll
                                for (int q4 = 0; q4 < HC / 4; q4++) {
                                    const int ml = tt * NTOK + half * HC + 4 * q4;
                                    pv[q4] = (tt < T && ml < un.len)
                                                 ? __ldcg(reinterpret_cast<const float4*>(part + (size_t)(ml / 4) * TROWS * 4))
                                                 : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                                }
#pragma unroll
                                for (int q4 = 0; q4 < HC / 4; q4++) {
                                    const float2 lo = make_float2(pv[q4].x, pv[q4].y), hi = make_float2(pv[q4].z, pv[q4].w);
                                    acc[tt][2 * q4] = c2 == 0 ? lo : __fadd2_rn(acc[tt][2 * q4], lo);
                                    acc[tt][2 * q4 + 1] = c2 == 0 ? hi : __fadd2_rn(acc[tt][2 * q4 + 1], hi);
                                }
                            }
                        }
                        float* out = sg.out;
#pragma unroll
                        for (int tt = 0; tt < TMAX; tt++) {
                            if (tt < T) {
#pragma unroll
                                for (int j = 0; j < HC; j++) {
                                    const int ml = tt * NTOK + half * HC + j;
                                    const int64_t m = un.m0 + ml;
                                    if (ml < un.len && m < args.m_out)
                                        out[m * sg.ldo + n] = j & 1 ? acc[tt][j / 2].y : acc[tt][j / 2].x;
                                }
                            }
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
    return (size_t)C::W_STAGES * C::TILE + (size_t)C::B_STAGES * C::B_STAGE + C::MINA + sizeof(GemmShared);
}

// Gather the requested canvas rows of a tiled activation into a compact tiled
// activation of Mp_r rows (rows past n_rows are zero).  One thread per 16-byte
// chunk: 16 quant chunks, 4 sums chunks and one scale per (super-block, row).
__global__ void gather_rows_kernel(const int8_t* __restrict__ q, const float* __restrict__ scale,
                                   const uint8_t* __restrict__ sums, int64_t M, int64_t Mp,
                                   const int32_t* __restrict__ rows, int32_t n_rows, int64_t Mp_r, int32_t nsb,
                                   int8_t* __restrict__ gq, float* __restrict__ gscale, uint8_t* __restrict__ gsums) {
    pdl_trigger();
    pdl_wait();
    const int64_t total = (int64_t)nsb * Mp_r * 21;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(g % 21);
        const int64_t i = (g / 21) % Mp_r;
        const int64_t s = g / 21 / Mp_r;
        int64_t m = -1;
        if (i < n_rows) {
            m = rows[i];
            if (m < 0 || m >= M) {
                if (c == 0) set_err(ERR_ROW_RANGE);
                m = -1;
            }
        }
        if (c < 16) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m >= 0)
                v = *reinterpret_cast<const uint4*>(q + ((s * (Mp / 8) + m / 8) * 16 + c) * 128 + (m % 8) * 16);
            *reinterpret_cast<uint4*>(gq + ((s * (Mp_r / 8) + i / 8) * 16 + c) * 128 + (i % 8) * 16) = v;
        } else if (c < 20) {
            const int cs = c - 16;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m >= 0)
                v = *reinterpret_cast<const uint4*>(sums + (s * (Mp / 8) + m / 8) * SUMS_GROUP + cs * 128 + (m % 8) * 16);
            *reinterpret_cast<uint4*>(gsums + (s * (Mp_r / 8) + i / 8) * SUMS_GROUP + cs * 128 + (i % 8) * 16) = v;
        } else {
            gscale[s * Mp_r + i] = m >= 0 ? scale[s * Mp + m] : 0.0f;
        }
    }
}

}  // namespace dllm
