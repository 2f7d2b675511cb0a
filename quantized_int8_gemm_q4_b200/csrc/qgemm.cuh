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
// Each plane sum stays within 2^22 in magnitude.  Each plane has its own int32
// accumulator in tensor memory, preset to the bit pattern of 1.5*2^23 (MAGIC): after
// a super-block's MMAs it holds the bits of the f32 1.5*2^23 + P exactly, so the
// epilogue needs no integer-to-float instruction.  It forms S with one FFMA and one
// FADD (packed f32x2), accumulates da * d * S in f32 registers, and writes the preset
// back before releasing the accumulator.
//
// The min term (Q4_K), on the tf32 tensor pipe.  Its per-super-block factor
// dmin[n] * da[m] is a product of a row term and a column term, so
//   -sum_sb da dmin Smin = sum over (sb, j) of (-dmin m_j)[n] * (da sum32_j)[m],
// a GEMM with one K step per sub-block.  Both operands are split as hi + lo with hi
// exact in tf32 (-dmin m_j is exact in hi + lo; da*sum32_j loses at most 2^-22 of
// itself), and hi*hi + hi*lo + lo*hi accumulate in an f32 tensor-memory accumulator
// over the whole K range of a work unit, read once per unit.  The dropped lo*lo
// product and the split lose at most 2^-21 of each product's magnitude; the f32
// accumulation over the unit's K/32 sub-block steps adds at most (K/32) * 2^-24 of
// the running sum of magnitudes (about 2^-17 at K = 4096); both bounds are relative to
// the min term's own sum of |terms|, a part of the 1e-6 * sum|terms| tolerance.
//
// Pipeline (16 warps, one CTA per SM, persistent over work units).  Per super-block
// the MMAs run plane-major: the 8 K-steps of plane 0 into accumulator P0, then the 8
// of plane 1 into P1, then (Q4_K) the 3 min-term MMAs.  Every MMA covers all of the
// unit's tokens (N <= 128; at N = 128 one int8 MMA takes ~64 cycles, the pipe's full
// rate).  So each plane accumulator is drained by the epilogue while the other plane's
// MMAs run, and the tensor pipe never waits for an epilogue hand-off.
//   warp 0      weight producer: bulk copies of weight tiles into a shared-memory
//               ring.  Weights are never written by the kernels this library chains
//               with programmatic dependent launch, so these copies start before the
//               dependency wait.
//   warp 1      MMA issuer of plane 0 (one thread) and tensor-memory allocation
//   warp 2      activation producer: bulk copies of activation tiles (int8 codes,
//               scales, scaled sums), after the dependency wait
//   warp 3      MMA issuer of plane 1 and of the min term (one thread)
//   warps 4-7   unpack, one group of four (UNPACK_GROUPS): thread = weight row; it
//               builds both quarter super-blocks (two K-steps each, both weight planes)
//               of every half super-block into a tensor-memory ring (the A operand), and
//               writes the min-term A operand (Q4_K) to shared memory and the f32 d.
//               A second group (20 warps, each group one quarter) measured slower: the
//               512-thread CTA leaves the issuers and the epilogue more issue slots.
//   warps 8-15  epilogue: two warps per tensor-memory lane quadrant, each on 64 of the
//               token columns
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
// Unpack groups of four warps (one warp per tensor-memory lane quadrant).  One group
// (a 512-thread CTA) measured faster than two: fewer warps contend for issue slots.
constexpr int UNPACK_GROUPS = 1;
constexpr int UNPACK_THREADS = 128 * UNPACK_GROUPS;
constexpr int EPI_WARP0 = 4 + 4 * UNPACK_GROUPS;  // first epilogue warp
constexpr int GEMM_THREADS = 128 + UNPACK_THREADS + 256;
constexpr int UNIT_TOKENS = 128;
constexpr int EPI_COLS = 64;                       // token columns per epilogue thread
constexpr int MAX_KC = 16;                         // K-chunks per tile, at most
constexpr int S_SLOTS = 4;                         // d ring (unpack -> epilogue)
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s
// Registers per thread of each warpgroup after setmaxnreg: producers and issuers (one
// warpgroup), unpack (two) and epilogue (two).  setmaxnreg.inc draws on the registers the
// CTA was launched with (its threads x the kernel's register count), so the split must
// not exceed them, or the increasing warps would wait for registers that never come
// free.  REG_LAUNCH_MIN is the launch count the split assumes; the host checks the
// compiled kernel's count against it before the first launch.
constexpr int REG_CTRL = 48, REG_UNPACK = 64, REG_EPI = UNPACK_GROUPS == 1 ? 200 : 152;
constexpr int REG_SPLIT_TOTAL = 128 * REG_CTRL + UNPACK_THREADS * REG_UNPACK + 256 * REG_EPI;
constexpr int REG_LAUNCH_MIN = 65536 / GEMM_THREADS / 8 * 8;
static_assert(REG_SPLIT_TOTAL <= GEMM_THREADS * REG_LAUNCH_MIN && GEMM_THREADS * REG_LAUNCH_MIN <= 65536,
              "register split over the launch budget");
static_assert(REG_CTRL % 8 == 0 && REG_UNPACK % 8 == 0 && REG_EPI % 8 == 0 && REG_CTRL >= 24, "setmaxnreg counts");

// Activation "sums" operand of one super-block: per 8-row group 512 bytes =
// [hi j0-3 | hi j4-7 | lo j0-3 | lo j4-7] x [8 rows x 16 bytes].
constexpr int SUMS_GROUP = 512;

// Tensor-memory columns: the A ring (A_SLOTS half super-blocks; a half is four K-steps
// of 16 columns, [plane 0: 8 | plane 1: 8]), then the plane accumulators P0 and P1 (128
// token columns each), then (Q4_K) the f32 min-term accumulator.
constexpr uint32_t TM_COLS = 512;
constexpr uint32_t TM_A = 0;

template <int QT>
struct GemmCfg;
template <>
struct GemmCfg<12> {  // Q4_K
    static constexpr int TILE = Q4K_TILE;
    static constexpr bool MIN = true;
    static constexpr int W_STAGES = 4;
    static constexpr int B_STAGES = 3;
    static constexpr int B_Q = UNIT_TOKENS * 256;
    static constexpr int B_SUMS = UNIT_TOKENS / 8 * SUMS_GROUP;
    static constexpr int B_STAGE = B_Q + B_SUMS + UNIT_TOKENS * 4;
    static constexpr int MINA = 2 * 4096;  // -dmin*m_j as [hi | lo], canonical K-major 128 rows x 32 B
    static constexpr int MINA_BUFS = 2;
    static constexpr int A_SLOTS = 2;      // one super-block
    static constexpr uint32_t TM_P0 = TM_A + 64 * A_SLOTS;
    static constexpr uint32_t TM_P1 = TM_P0 + UNIT_TOKENS;
    static constexpr uint32_t TM_MIN = TM_P1 + UNIT_TOKENS;
    static constexpr uint32_t TM_END = TM_MIN + UNIT_TOKENS;
};
template <>
struct GemmCfg<14> {  // Q6_K
    static constexpr int TILE = Q6K_TILE;
    static constexpr bool MIN = false;
    static constexpr int W_STAGES = 4;
    static constexpr int B_STAGES = 3;
    static constexpr int B_Q = UNIT_TOKENS * 256;
    static constexpr int B_SUMS = 0;
    static constexpr int B_STAGE = B_Q + B_SUMS + UNIT_TOKENS * 4;
    static constexpr int MINA = 0;
    static constexpr int MINA_BUFS = 0;
    static constexpr int A_SLOTS = 4;      // two super-blocks: the unpack runs one ahead
    static constexpr uint32_t TM_P0 = TM_A + 64 * A_SLOTS;
    static constexpr uint32_t TM_P1 = TM_P0 + UNIT_TOKENS;
    static constexpr uint32_t TM_MIN = 0;
    static constexpr uint32_t TM_END = TM_P1 + UNIT_TOKENS;
};
static_assert(GemmCfg<12>::TM_END <= TM_COLS && GemmCfg<14>::TM_END <= TM_COLS, "tensor-memory columns over budget");

// K-step (of 32) that sub-position kk of quarter q holds.  Q4_K: the quarter is one
// 32-byte nibble chunk, K-steps 2q (low nibbles) and 2q+1 (high nibbles).  Q6_K: the
// two K-steps that share their low-bit bytes, 4h + g and 4h + g + 2 (h = q/2, g = q%2).
template <int QT>
__host__ __device__ constexpr int kstep_of(int q, int kk) {
    return QT == 12 ? 2 * q + kk : 4 * (q >> 1) + (q & 1) + 2 * kk;
}

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
    int32_t nsb;       // weight super-blocks per row (K / 256; 2K / 256 for Q5_K's split form)
    int32_t nsb_act;   // activation super-blocks per row: weight super-block s reads s % nsb_act
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
    int32_t stall;     // test: the producers issue nothing, so every other role's wait runs out
    int64_t dbg_N;
};

struct GemmShared {
    uint64_t w_full[4], w_empty[4];
    uint64_t b_full[3], b_empty[3];
    uint64_t a_full[4], a_empty[4];   // A ring slots: half super-blocks
    uint64_t p_full[2], p_empty[2];   // plane accumulators P0, P1
    uint64_t m_full[2], m_empty[2];   // min-term A operand buffers (Q4_K)
    uint64_t min_full, min_empty;     // min-term accumulator (Q4_K), once per unit
    uint64_t s_full[S_SLOTS], s_empty[S_SLOTS];
    uint64_t final_bar;
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
// Drain wait of an aborting CTA: waits for the CTA's own asynchronous work (bulk copies
// into its shared memory, MMAs on its tensor memory) regardless of the abort flag,
// bounded by its own limit.  True if the phase completed.
__device__ __forceinline__ bool drain_bar(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 200000u)) {
        if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            set_err(ERR_TIMEOUT);
            return false;
        }
    }
    return true;
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

// 64 consecutive accumulator columns of this warp's 32 lanes.
__device__ __forceinline__ void load_cols64(uint32_t taddr, uint32_t (&x)[EPI_COLS]) {
    tmem_ld16(taddr, x);
    tmem_ld16(taddr + 16, x + 16);
    tmem_ld16(taddr + 32, x + 32);
    tmem_ld16(taddr + 48, x + 48);
}
// Write the MAGIC preset into 64 consecutive accumulator columns of this warp's lanes.
__device__ __forceinline__ void preset_cols64(uint32_t taddr) {
    uint32_t m[16];
#pragma unroll
    for (int i = 0; i < 16; i++) m[i] = MAGIC_BITS;
    tmem_st16(taddr, m);
    tmem_st16(taddr + 16, m);
    tmem_st16(taddr + 32, m);
    tmem_st16(taddr + 48, m);
}

// Store the first cnt of this thread's EPI_COLS accumulated outputs: column j goes to
// p + j * ld (one output row per token; the warp's 32 lanes are 32 consecutive n).
__device__ __forceinline__ void store_cols(float* p, int64_t ld, int cnt, const float2 (&acc)[EPI_COLS / 2]) {
#pragma unroll
    for (int j = 0; j < EPI_COLS; j++) {
        if (j < cnt) *p = j & 1 ? acc[j / 2].y : acc[j / 2].x;
        p += ld;
    }
}

template <int QT, bool DBG, bool TAIL>
__global__ void __launch_bounds__(GEMM_THREADS, 1) qgemm_kernel(const __grid_constant__ GemmArgs args) {
    using C = GemmCfg<QT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* w_stage = smem_raw;
    uint8_t* b_stage = w_stage + C::W_STAGES * C::TILE;
    uint8_t* mina = b_stage + C::B_STAGES * C::B_STAGE;
    GemmShared& sh = *reinterpret_cast<GemmShared*>(mina + C::MINA_BUFS * C::MINA);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_units = args.n_units;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::W_STAGES; i++) { mbar_init(&sh.w_full[i], 1); mbar_init(&sh.w_empty[i], UNPACK_THREADS); }
        // an activation stage is released by a commit from each issuer (their MMAs are
        // done) and by the 256 epilogue threads (the scales are read)
        for (int i = 0; i < C::B_STAGES; i++) { mbar_init(&sh.b_full[i], 1); mbar_init(&sh.b_empty[i], 258); }
        for (int i = 0; i < C::A_SLOTS; i++) { mbar_init(&sh.a_full[i], UNPACK_THREADS); mbar_init(&sh.a_empty[i], 2); }
        for (int i = 0; i < 2; i++) { mbar_init(&sh.p_full[i], 1); mbar_init(&sh.p_empty[i], 256); }
        for (int i = 0; i < 2; i++) { mbar_init(&sh.m_full[i], 128); mbar_init(&sh.m_empty[i], 1); }
        mbar_init(&sh.min_full, 1);
        mbar_init(&sh.min_empty, 256);
        for (int i = 0; i < S_SLOTS; i++) { mbar_init(&sh.s_full[i], 128); mbar_init(&sh.s_empty[i], 256); }
        mbar_init(&sh.final_bar, 2);
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
    // Everything above, and the weight copies, may overlap the previous kernel on the
    // stream; every access to global memory that earlier work can write comes after
    // pdl_wait in the role that makes it.
    if (threadIdx.x == 0) pdl_trigger();

    if (warp < 4) {
        setmaxnreg_dec<REG_CTRL>();
        if (warp == 0 || warp == 2) {
            // ======================================================== producers
            // warp 0: weight tiles; warp 2: activation tiles.  A thread keeps only one bulk
            // copy in flight at a time (its copies run one after another, each costing a
            // full memory latency), so every ring stage has lanes of its own: weight
            // stage i is lane i; activation stage i is lanes 3i (codes; it also arms the
            // barrier with the stage's byte count), 3i+1 (scaled sums, Q4_K) and 3i+2
            // (scales).  The lanes of one stage agree on each wait, so they issue all of a
            // stage's copies or none.
            const bool wprod = warp == 0;
            const int NST = wprod ? C::W_STAGES : C::B_STAGES;
            const int st = wprod ? lane : lane / 3;
            const int part = wprod ? 0 : lane % 3;
            const bool active = st < NST && (wprod || C::B_SUMS || part != 1);
            const uint32_t smask = wprod ? 0u : (C::B_SUMS ? 7u : 5u) << (3 * st);
            uint64_t* full = wprod ? sh.w_full : sh.b_full;
            uint64_t* empty = wprod ? sh.w_empty : sh.b_empty;
            uint32_t ph = 0;
            bool inflight = false;  // a copy of this lane's stage has been issued and not waited for
            if (!wprod) pdl_wait();
            if (active) {
                const uint64_t pol = wprod ? policy_evict_first() : policy_evict_last();
                const int64_t n_prod = args.stall ? 0 : n_units;
                uint32_t g = 0;  // super-blocks of this CTA so far
                for (int64_t u = blockIdx.x; u < n_prod; u += gridDim.x) {
                    const Unit un = unit_of<TAIL>(args, u);
                    const uint8_t* wt = args.seg[un.seg].w + (size_t)un.tile * args.nsb * C::TILE;
                    for (int s = un.sb0; s < un.sb1; s++, g++) {
                        if ((int)(g % NST) != st) continue;
                        bool ok = wait_bar(sh, &empty[st], ph ^ 1);
                        if (!wprod) ok = __all_sync(smask, ok);
                        if (!ok) goto prod_done;
                        if (wprod) {
                            mbar_arrive_expect_tx(&full[st], C::TILE);
                            bulk_g2s_hint(w_stage + st * C::TILE, wt + (size_t)s * C::TILE, C::TILE, &full[st], pol);
                        } else {
                            uint8_t* bs = b_stage + st * C::B_STAGE;
                            const int64_t t0 = un.m0;
                            const int64_t sa = s % args.nsb_act;  // activation super-block
                            const uint32_t ntok = (uint32_t)un.len;
                            const uint32_t sums_bytes = C::B_SUMS ? ntok / 8 * SUMS_GROUP : 0;
                            if (part == 0) mbar_arrive_expect_tx(&full[st], ntok * 256 + sums_bytes + ntok * 4);
                            __syncwarp(smask);  // the stage's byte count is armed before any of its copies lands
                            if (part == 0)
                                bulk_g2s_hint(bs, args.q + ((size_t)sa * args.Mp + t0) * 256, ntok * 256, &full[st], pol);
                            else if (part == 1)
                                bulk_g2s_hint(bs + C::B_Q, args.sums + ((size_t)sa * args.Mp + t0) / 8 * SUMS_GROUP,
                                              sums_bytes, &full[st], pol);
                            else
                                bulk_g2s_hint(bs + C::B_Q + C::B_SUMS, args.scale + (size_t)sa * args.Mp + t0, ntok * 4,
                                              &full[st], pol);
                        }
                        inflight = true;
                        ph ^= 1;
                    }
                }
            }
        prod_done:
            // never leave with bulk copies in flight into this CTA's shared memory: the
            // stage's last phase completes once every copy of it has landed
            if (sh.abort_flag && inflight && (wprod || part == 0)) (void)drain_bar(&full[st], ph ^ 1);
        } else {
            // ======================================================== MMA issuers
            // One thread issues a tcgen05 instruction only every ~50-100 cycles, about
            // the time an N = 128 int8 MMA takes, so the work is split between two warps:
            // warp 1 issues plane 0 into P0; warp 3 issues plane 1 into P1 and the
            // min-term MMAs.  Both read the same A-ring halves and activation stage, so
            // each of those is released by a commit from each issuer.
            const bool leader = lane == 0;
            const int plane = warp == 1 ? 0 : 1;
            constexpr uint32_t ASG = QT == 12 ? 0 : 1;  // plane operand type: u8 (Q4_K), s8 (Q6_K)
            uint32_t sbc = 0, uc = 0;
            for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, uc++) {
                const Unit un = unit_of<TAIL>(args, u);
                const uint32_t ntok = (uint32_t)un.len;
                const uint32_t id = idesc_i8(128, (int)ntok, (int)ASG, 1);
                for (int s = un.sb0; s < un.sb1; s++, sbc++) {
                    const uint32_t bst = sbc % C::B_STAGES;
                    if (!wait_bar_warp(sh, &sh.b_full[bst], (sbc / C::B_STAGES) & 1)) goto mma_done;
                    // this plane's accumulator has been drained and preset by the epilogue
                    if (!wait_bar_warp(sh, &sh.p_empty[plane], sbc & 1)) goto mma_done;
                    const uint32_t stg = smem_u32(b_stage + bst * C::B_STAGE);
                    const uint64_t bdesc = sdesc_kmajor_noswz(stg, 128, 2048);
#pragma unroll 1
                    for (int hh = 0; hh < 2; hh++) {
                        const uint32_t hc = 2 * sbc + hh, sl = hc % C::A_SLOTS;
                        if (!wait_bar_warp(sh, &sh.a_full[sl], (hc / C::A_SLOTS) & 1)) goto mma_done;
                        tc_fence_after();
                        if (leader) {
#pragma unroll
                            for (int kq = 0; kq < 4; kq++) {
                                const int q = 2 * hh + (kq >> 1), kk = kq & 1;
                                mma_i8_ts(tmem + (plane ? C::TM_P1 : C::TM_P0), tmem + TM_A + 64 * sl + 16 * kq + 8 * plane,
                                          bdesc + 16 * kstep_of<QT>(q, kk), id, 1u);
                            }
                            tc_commit(&sh.a_empty[sl]);
                        }
                        __syncwarp();
                    }
                    if (leader) tc_commit(&sh.p_full[plane]);
                    __syncwarp();
                    if constexpr (C::MIN) {
                        if (plane == 1) {
                            // ---- min term: (-dmin m_j) x (da sum32_j), three tf32 products
                            const uint32_t mb = sbc & 1;
                            if (!wait_bar_warp(sh, &sh.m_full[mb], (sbc >> 1) & 1)) goto mma_done;
                            // a unit's first min-term MMA overwrites the accumulator: the
                            // previous unit's epilogue must have read it out
                            if (s == un.sb0 && !wait_bar_warp(sh, &sh.min_empty, (uc & 1) ^ 1)) goto mma_done;
                            tc_fence_after();
                            if (leader) {
                                const uint32_t idm = idesc_tf32(128, (int)ntok);
                                const uint32_t ma = smem_u32(mina + mb * C::MINA);
                                const uint64_t a_hi = sdesc_kmajor_noswz(ma, 128, 256);
                                const uint64_t a_lo = sdesc_kmajor_noswz(ma + 4096, 128, 256);
                                const uint64_t b_hi = sdesc_kmajor_noswz(stg + C::B_Q, 128, SUMS_GROUP);
                                const uint64_t b_lo = sdesc_kmajor_noswz(stg + C::B_Q + 256, 128, SUMS_GROUP);
                                mma_tf32_ss(tmem + C::TM_MIN, a_hi, b_hi, idm, s > un.sb0 ? 1u : 0u);
                                mma_tf32_ss(tmem + C::TM_MIN, a_hi, b_lo, idm, 1u);
                                mma_tf32_ss(tmem + C::TM_MIN, a_lo, b_hi, idm, 1u);
                                tc_commit(&sh.m_empty[mb]);
                                if (s == un.sb1 - 1) tc_commit(&sh.min_full);
                            }
                            __syncwarp();
                        }
                    }
                    if (leader) tc_commit(&sh.b_empty[bst]);
                    __syncwarp();
                }
            }
        mma_done:
            // every MMA this warp issued has completed before tensor memory is freed (the
            // barrier takes one commit from each issuer)
            if (leader) tc_commit(&sh.final_bar);
            __syncwarp();
            (void)drain_bar(&sh.final_bar, 0);
            __syncwarp();
        }
    } else if (warp < EPI_WARP0) {
        setmaxnreg_dec<REG_UNPACK>();
        // ============================================================ unpack
        // Two groups of four warps (one warp per lane quadrant each).  Per super-block
        // both decode this row's scales; group 0 hands d to the epilogue and (Q4_K) the
        // min-term A operand to the issuer.  In each half super-block, group g builds the
        // two weight planes of quarter 2*half + g (two K-steps); the half is published
        // once both groups have stored theirs.
        const int quad = warp & 3;
        const int grp = (warp - 4) >> 2;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        uint32_t ws = 0, wph = 0, ss = 0, sph = 0, sbc = 0;
        for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
            const Unit un = unit_of<TAIL>(args, u);
            for (int s = un.sb0; s < un.sb1; s++, sbc++) {
                if (!wait_bar_warp(sh, &sh.w_full[ws], wph)) goto unpack_done;
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
                    if (grp == 0) {
                        if (!wait_bar_warp(sh, &sh.s_empty[ss], sph ^ 1)) goto unpack_done;
                        sh.dd[ss][row] = d;
                        mbar_arrive(&sh.s_full[ss]);
                        if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
                        // -dmin*m_j as tf32 hi + lo: row `row` of the canonical K-major layout
                        // (8-row groups of 256 bytes, two 16-byte K chunks)
                        const uint32_t mb = sbc & 1;
                        if (!wait_bar_warp(sh, &sh.m_empty[mb], ((sbc >> 1) & 1) ^ 1)) goto unpack_done;
                        float hi[8], lo[8];
#pragma unroll
                        for (int j = 0; j < 8; j++) split_tf32(nmin[j], hi[j], lo[j]);
                        uint8_t* base = mina + mb * C::MINA + (row >> 3) * 256 + (row & 7) * 16;
                        *reinterpret_cast<float4*>(base) = make_float4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<float4*>(base + 128) = make_float4(hi[4], hi[5], hi[6], hi[7]);
                        *reinterpret_cast<float4*>(base + 4096) = make_float4(lo[0], lo[1], lo[2], lo[3]);
                        *reinterpret_cast<float4*>(base + 4096 + 128) = make_float4(lo[4], lo[5], lo[6], lo[7]);
                        fence_proxy_async_smem();
                        mbar_arrive(&sh.m_full[mb]);
                    }
#pragma unroll 1
                    for (int hh = 0; hh < 2; hh++) {
                        const uint32_t hc = 2 * sbc + hh, sl = hc % C::A_SLOTS;
                        if (!wait_bar_warp(sh, &sh.a_empty[sl], ((hc / C::A_SLOTS) & 1) ^ 1)) goto unpack_done;
#pragma unroll
                        for (int gq = grp; gq < 2; gq += UNPACK_GROUPS) {
                        const int q = 2 * hh + gq;
                        // 32-byte quant chunk q: sub-block 2q in the low nibbles, 2q+1 in the high
                        const uint4 p0 = *reinterpret_cast<const uint4*>(tl + ((2 * q) * TROWS + row) * 16);
                        const uint4 p1 = *reinterpret_cast<const uint4*>(tl + ((2 * q + 1) * TROWS + row) * 16);
                        const uint32_t wv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                        const uint32_t sca = q == 0 ? sc[0] : q == 1 ? sc[2] : q == 2 ? sc[4] : sc[6];
                        const uint32_t scb = q == 0 ? sc[1] : q == 1 ? sc[3] : q == 2 ? sc[5] : sc[7];
#pragma unroll
                        for (int kk = 0; kk < 2; kk++) {
                            const uint32_t s6 = kk ? scb : sca;
                            const uint32_t lo3 = s6 & 7, hi3 = s6 >> 3;
                            uint32_t v[16];
#pragma unroll
                            for (int i = 0; i < 8; i++) {
                                const uint32_t nib = (wv[i] >> (4 * kk)) & 0x0F0F0F0Fu;
                                v[i] = nib * lo3;
                                v[8 + i] = nib * hi3;
                            }
                            tmem_st16(tmem + lane_off + TM_A + 64 * sl + 32 * gq + 16 * kk, v);
                        }
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sh.a_full[sl]);
                    }
                } else {
                    const uint4 scv = *reinterpret_cast<const uint4*>(tl + Q6K_OFF_SC + 16 * row);
                    const uint32_t scw[4] = {scv.x, scv.y, scv.z, scv.w};
                    const float d = __half2float(
                        __ushort_as_half(*reinterpret_cast<const unsigned short*>(tl + Q6K_OFF_D + 2 * row)));
                    if (grp == 0) {
                        if (!wait_bar_warp(sh, &sh.s_empty[ss], sph ^ 1)) goto unpack_done;
                        sh.dd[ss][row] = d;
                        mbar_arrive(&sh.s_full[ss]);
                        if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
                    }
#pragma unroll 1
                    for (int hh = 0; hh < 2; hh++) {
                        const uint32_t hc = 2 * sbc + hh, sl = hc % C::A_SLOTS;
                        if (!wait_bar_warp(sh, &sh.a_empty[sl], ((hc / C::A_SLOTS) & 1) ^ 1)) goto unpack_done;
#pragma unroll 1
                        for (int gq = grp; gq < 2; gq += UNPACK_GROUPS) {
                        const int q = 2 * hh + gq;
                        // K-steps 4h + g and 4h + g + 2 share their low-bit bytes (low and high
                        // nibbles) and the half's high-bit bytes
                        const int h = q >> 1, g = q & 1;
                        const int lp = 2 * (2 * h + g);  // low-bit piece index
                        const uint4 l0 = *reinterpret_cast<const uint4*>(tl + (lp * TROWS + row) * 16);
                        const uint4 l1 = *reinterpret_cast<const uint4*>(tl + ((lp + 1) * TROWS + row) * 16);
                        const uint4 h0 =
                            *reinterpret_cast<const uint4*>(tl + Q6K_OFF_QH + ((2 * h) * TROWS + row) * 16);
                        const uint4 h1 =
                            *reinterpret_cast<const uint4*>(tl + Q6K_OFF_QH + ((2 * h + 1) * TROWS + row) * 16);
                        const uint32_t lw[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
                        const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                        // scale bytes 2ks, 2ks+1 of K-step ks = 4h + g + 2kk sit in word 2h + kk at
                        // bit offset 16g
                        const uint32_t swq[2] = {h ? scw[2] : scw[0], h ? scw[3] : scw[1]};
#pragma unroll
                        for (int kk = 0; kk < 2; kk++) {
                            const int G = g + 2 * kk;
                            const int sh_lo = 4 * kk, sh_hi = 2 * G;
                            const int32_t sca = (int32_t)(int8_t)((swq[kk] >> (16 * g)) & 0xFF);
                            const int32_t scb = (int32_t)(int8_t)((swq[kk] >> (16 * g + 8)) & 0xFF);
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
                            tmem_st16(tmem + lane_off + TM_A + 64 * sl + 32 * gq + 16 * kk, v);
                        }
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sh.a_full[sl]);
                    }
                }
                mbar_arrive(&sh.w_empty[ws]);
                if (++ws == C::W_STAGES) { ws = 0; wph ^= 1; }
            }
        }
    unpack_done:;
    } else {
        setmaxnreg_inc<REG_EPI>();
        // ============================================================ epilogue
        const int quad = warp & 3;
        const int half = (warp - EPI_WARP0) >> 2;
        const int row = quad * 32 + lane;
        const int etid = threadIdx.x - (128 + UNPACK_THREADS);  // 0..255
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t col0 = (uint32_t)(half * EPI_COLS);
        // initial preset of both plane accumulators (this warp's lanes and columns)
        preset_cols64(tmem + lane_off + C::TM_P0 + col0);
        preset_cols64(tmem + lane_off + C::TM_P1 + col0);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.p_empty[0]);
        mbar_arrive(&sh.p_empty[1]);
        pdl_wait();  // outputs, partials and counters may be in use by earlier work
        // plane 1 carries weight 8 (Q4_K) or 256 (Q6_K): kP * (M + P1) - kP * M = kP * P1
        const float2 kP = QT == 12 ? make_float2(8.0f, 8.0f) : make_float2(256.0f, 256.0f);
        const float2 nkM = QT == 12 ? make_float2(-8.0f * MAGIC, -8.0f * MAGIC)
                                    : make_float2(-256.0f * MAGIC, -256.0f * MAGIC);
        const float2 nM = make_float2(-MAGIC, -MAGIC);
        uint32_t ss = 0, sph = 0, sbc = 0, uc = 0, epi_ph = 0;
        for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, uc++) {
            int sb_first, sb_end, ulen;
            {
                const Unit u0 = unit_of<TAIL>(args, u);
                sb_first = u0.sb0;
                sb_end = u0.sb1;
                ulen = u0.len;
            }
            const bool live = (int)col0 < ulen;  // this thread has token columns in the unit
            float2 acc[EPI_COLS / 2];
#pragma unroll
            for (int j = 0; j < EPI_COLS / 2; j++) acc[j] = make_float2(0.0f, 0.0f);
            for (int s = sb_first; s < sb_end; s++, sbc++) {
                const uint32_t bst = sbc % C::B_STAGES;
                if (!wait_bar_warp(sh, &sh.s_full[ss], sph)) goto epi_done;
                const float dv = sh.dd[ss][row];
                mbar_arrive(&sh.s_empty[ss]);
                if (++ss == S_SLOTS) { ss = 0; sph ^= 1; }
                const float2 d2 = make_float2(dv, dv);
                if (!wait_bar_warp(sh, &sh.b_full[bst], (sbc / C::B_STAGES) & 1)) goto epi_done;
                const float* da = reinterpret_cast<const float*>(b_stage + bst * C::B_STAGE + C::B_Q + C::B_SUMS) + col0;
                if constexpr (DBG) {
                    // the integer S of every element: both planes, exactly
                    uint32_t x0[EPI_COLS];
                    if (!wait_bar_warp(sh, &sh.p_full[0], sbc & 1)) goto epi_done;
                    tc_fence_after();
                    if (live) {
                        load_cols64(tmem + lane_off + C::TM_P0 + col0, x0);
                        tmem_wait_ld();
                        preset_cols64(tmem + lane_off + C::TM_P0 + col0);
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    mbar_arrive(&sh.p_empty[0]);
                    if (!wait_bar_warp(sh, &sh.p_full[1], sbc & 1)) goto epi_done;
                    tc_fence_after();
                    if (live) {
                        const Unit un = unit_of<TAIL>(args, u);
#pragma unroll
                        for (int c = 0; c < 4; c++) {
                            uint32_t x1[16];
                            tmem_ld16(tmem + lane_off + C::TM_P1 + col0 + 16 * c, x1);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; i++) {
                                const int ml = (int)col0 + 16 * c + i;
                                const int64_t m = un.m0 + ml;
                                if (ml < un.len && m < args.m_out) {
                                    const int64_t n = un.tile * TROWS + row;
                                    const int32_t P0 = (int32_t)(x0[16 * c + i] - MAGIC_BITS);
                                    const int32_t P1 = (int32_t)(x1[i] - MAGIC_BITS);
                                    args.dbg_S[(m * args.dbg_N + n) * args.nsb + s] = P0 + (QT == 12 ? 8 : 256) * P1;
                                }
                            }
                        }
                        preset_cols64(tmem + lane_off + C::TM_P1 + col0);
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    mbar_arrive(&sh.p_empty[1]);
                } else {
                    // each plane on its own: acc += da * d * (weight of the plane) * P, where
                    // P comes exactly out of the f32 1.5*2^23 + P; two chunks of 32 columns
#pragma unroll
                    for (int pl = 0; pl < 2; pl++) {
                        if (!wait_bar_warp(sh, &sh.p_full[pl], sbc & 1)) goto epi_done;
                        tc_fence_after();
                        if (live) {
                            const uint32_t tp = tmem + lane_off + (pl ? C::TM_P1 : C::TM_P0) + col0;
#pragma unroll
                            for (int c = 0; c < 2; c++) {
                                uint32_t x[32];
                                tmem_ld16(tp + 32 * c, x);
                                tmem_ld16(tp + 32 * c + 16, x + 16);
                                tmem_wait_ld();
#pragma unroll
                                for (int i4 = 0; i4 < 8; i4++) {
                                    const float4 dv4 = *reinterpret_cast<const float4*>(da + 32 * c + 4 * i4);
#pragma unroll
                                    for (int h2 = 0; h2 < 2; h2++) {
                                        const int i = 2 * i4 + h2;
                                        const float2 X = make_float2(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
                                        const float2 T = pl ? __ffma2_rn(X, kP, nkM) : __fadd2_rn(X, nM);
                                        const float2 dd = __fmul2_rn(d2, h2 ? make_float2(dv4.z, dv4.w)
                                                                            : make_float2(dv4.x, dv4.y));
                                        acc[16 * c + i] = __ffma2_rn(T, dd, acc[16 * c + i]);
                                    }
                                }
                            }
                            preset_cols64(tp);
                            tmem_wait_st();
                        }
                        tc_fence_before();
                        mbar_arrive(&sh.p_empty[pl]);
                    }
                }
                mbar_arrive(&sh.b_empty[bst]);
            }
            if constexpr (C::MIN) {
                // the unit's min-term accumulator, complete once min_full flips
                if (!wait_bar_warp(sh, &sh.min_full, uc & 1)) goto epi_done;
                tc_fence_after();
                if (live) {
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        uint32_t y[16];
                        tmem_ld16(tmem + lane_off + C::TM_MIN + col0 + 16 * c, y);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 8; i++)
                            acc[8 * c + i] = __fadd2_rn(acc[8 * c + i],
                                                        make_float2(__uint_as_float(y[2 * i]), __uint_as_float(y[2 * i + 1])));
                    }
                }
                tc_fence_before();
                mbar_arrive(&sh.min_empty);
            }
            if constexpr (!DBG) {
                const Unit un = unit_of<TAIL>(args, u);
                const Segment& sg = args.seg[un.seg];
                const int64_t n = un.tile * TROWS + row;
                // uniform split: every tile has kc pieces and partial slots are unit indices
                const int np = TAIL ? un.np : args.kc;
                // output rows of this thread: canvas rows m0 + col0 + j for j < cnt
                const int64_t mfirst = un.m0 + col0;
                const int cnt = (int)min((int64_t)min(EPI_COLS, un.len - (int)col0), args.m_out - mfirst);
                if (np == 1) {
                    if (cnt > 0) store_cols(sg.out + mfirst * sg.ldo + n, sg.ldo, cnt, acc);
                } else {
                    // this K-chunk's partial: [unit][mu/4][128 rows][4 tokens], so a thread's
                    // 4 consecutive tokens are one 16-byte store and a warp's 32 rows 512
                    // contiguous bytes (token counts are multiples of 16)
                    const int64_t my_slot = TAIL ? un.slot0 + (int64_t)un.chunk * un.pstride : u;
                    float* part = args.partials + (size_t)my_slot * args.mu * TROWS + row * 4;
#pragma unroll
                    for (int q4 = 0; q4 < EPI_COLS / 4; q4++) {
                        const int ml = (int)col0 + 4 * q4;
                        if (ml < un.len)
                            __stcg(reinterpret_cast<float4*>(part + (size_t)(ml / 4) * TROWS * 4),
                                   make_float4(acc[2 * q4].x, acc[2 * q4].y, acc[2 * q4 + 1].x, acc[2 * q4 + 1].y));
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
                    if (sh.last_flag && live) {
                        // sum the piece partials in piece order.  Per 16-column group, up to
                        // four pieces' loads (16 x 16 bytes) are in flight together: each
                        // batch costs one L2 round trip.
#pragma unroll
                        for (int c4 = 0; c4 < EPI_COLS / 16; c4++) {
#pragma unroll 1
                            for (int c2b = 0; c2b < np; c2b += 4) {
                                float4 pv[4][4];
#pragma unroll
                                for (int k = 0; k < 4; k++) {
                                    const int c2 = c2b + k;
                                    const int64_t slot =
                                        TAIL ? un.slot0 + (int64_t)c2 * un.pstride : u - un.chunk + c2;
                                    const float* pp = args.partials + (size_t)slot * args.mu * TROWS + row * 4;
#pragma unroll
                                    for (int q4 = 0; q4 < 4; q4++) {
                                        const int ml = (int)col0 + 16 * c4 + 4 * q4;
                                        pv[k][q4] = c2 < np && ml < un.len
                                                        ? __ldcg(reinterpret_cast<const float4*>(pp + (size_t)(ml / 4) * TROWS * 4))
                                                        : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                                    }
                                }
#pragma unroll
                                for (int k = 0; k < 4; k++) {
                                    const int c2 = c2b + k;
                                    if (c2 < np) {
#pragma unroll
                                        for (int q4 = 0; q4 < 4; q4++) {
                                            const int a2 = 8 * c4 + 2 * q4;
                                            const float2 lo = make_float2(pv[k][q4].x, pv[k][q4].y);
                                            const float2 hi = make_float2(pv[k][q4].z, pv[k][q4].w);
                                            acc[a2] = c2 == 0 ? lo : __fadd2_rn(acc[a2], lo);
                                            acc[a2 + 1] = c2 == 0 ? hi : __fadd2_rn(acc[a2 + 1], hi);
                                        }
                                    }
                                }
                            }
                        }
                        if (cnt > 0) store_cols(sg.out + mfirst * sg.ldo + n, sg.ldo, cnt, acc);
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
    return (size_t)C::W_STAGES * C::TILE + (size_t)C::B_STAGES * C::B_STAGE + (size_t)C::MINA_BUFS * C::MINA +
           sizeof(GemmShared);
}
static_assert(gemm_smem_bytes<12>() <= 232448 && gemm_smem_bytes<14>() <= 232448, "shared memory over budget");

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
