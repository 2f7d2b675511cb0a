// Activation quantization fused with the step that produces its input in a forward
// pass (Architecture page, "A forward pass", steps 2 and 4): RMSNorm in front of the
// Q/K/V, gate/up and output projections, and the SwiGLU gate SiLU(g) * u in front of
// the down projection.  The f32 value each step produces is quantized in registers
// and never written to memory; the outputs are those of quantize_act_kernel, in the
// same layouts, so the GEMM consumes them unchanged.
//
// Precision: the normalised or gated value is formed in fp64 with explicitly rounded
// operations (no contraction) and rounded to f32 once; that f32 is quantized with
// quantize_act_kernel's arithmetic.  RMSNorm: ss = sum of x^2, r = 1/sqrt(ss/K + eps),
// y = f32((x * r) * gamma).  SwiGLU: h = f32((g / (1 + exp(-g))) * u).
#pragma once

#include "layout.cuh"

namespace dllm {

// Quantizes the 8 values v[] that this lane holds of one 256-block (elements
// 8 lane .. 8 lane + 7 of super-block s of canvas row m) and stores the codes, the
// block scale and the two-float scaled sub-block sums in the layouts that
// quantize_act_kernel writes (Mp = the canvas rounded up to 16 rows).  The whole warp
// calls it for the same (m, s).  Arithmetic: amax by warp reduction, iscale = 127/amax
// and scale = amax/127 as IEEE f32 divisions, code = round-half-even(v * iscale)
// clamped to [-127, 127]; sum of each sub-block of 32 (lanes 4j..4j+3) times scale.
__device__ __forceinline__ void quantize_store_lane(const float (&v)[8], int lane, int64_t m, int64_t s,
                                                    int64_t Mp, int8_t* __restrict__ q,
                                                    float* __restrict__ scale, uint8_t* __restrict__ sums) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i++) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float iscale = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    const float sc = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
    uint32_t packed[2] = {0u, 0u};
    int part = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        int t = __float2int_rn(__fmul_rn(v[i], iscale));
        t = max(-127, min(127, t));
        part += t;
        packed[i >> 2] |= (uint32_t)(t & 255) << (8 * (i & 3));
    }
    const int64_t g = m >> 3;
    const int r = (int)(m & 7);
    const int64_t blk = s * (Mp / 8) + g;
    // 16-byte chunk lane/2 of row r: [blk][chunk][8 rows][16 bytes], lane half (lane & 1)
    *reinterpret_cast<uint2*>(q + (blk * 16 + (lane >> 1)) * 128 + r * 16 + (lane & 1) * 8) =
        make_uint2(packed[0], packed[1]);
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if ((lane & 3) == 0) {
        const int j = lane >> 2;
        float hi, lo;
        split_tf32(__fmul_rn(sc, (float)part), hi, lo);
        float* ts = reinterpret_cast<float*>(sums + blk * 512);
        ts[((j >> 2) * 8 + r) * 4 + (j & 3)] = hi;
        ts[((2 + (j >> 2)) * 8 + r) * 4 + (j & 3)] = lo;
    }
    if (lane == 0) scale[s * Mp + m] = sc;
}

__device__ __forceinline__ void load8(const float* __restrict__ p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int FUSE_WARPS = 8;

// RMSNorm + quantize.  One CTA per output row m in [0, Mp) with W <= MAXW warps (the
// host picks the form: one super-block per warp up to 12 rows per SM, else up to 4 per
// warp in CTAs of at most 4 warps, so that six rows are in flight on each SM); warp w
// handles super-blocks w, w + W, ...  Output row m reads
// canvas row rows[m] when a row list is given (M is then the list's length and M_src the
// canvas height), else canvas row m.  The sum of squares is fp64 in one order whatever
// the form (so a row list gives the full canvas's rows bit for bit): per super-block,
// each lane's 8 squares in element order and then a butterfly over the 32 lanes; then,
// over the super-blocks, slot l = sum of the super-blocks l, l + 32, ... in that order
// (zero past the last) and a butterfly over the 32 slots.  Pass 1 keeps the warp's first
// SBR super-blocks of x in registers (and, with SBR = 1, the gamma of its super-block);
// pass 2 normalises and quantizes from them (the wide form reads gamma, the same for
// every row, from L1 there), re-reading only super-blocks beyond those
// (K > SBR * W * 256).  Rows M..Mp-1, and rows whose list entry is outside [0, M_src),
// are written as zeros; the latter also set ERR_ROW_RANGE.
constexpr int RMS_MAX_WARPS = 32;
constexpr int RMS_MAX_SB = 256;  // K <= 65536

__device__ __forceinline__ double butterfly_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ double squares8(const float (&v)[8]) {
    double ps = 0.0;
#pragma unroll
    for (int i = 0; i < 8; i++) ps = __dadd_rn(ps, __dmul_rn((double)v[i], (double)v[i]));
    return ps;
}

template <int SBR, int MAXW>
__global__ void __launch_bounds__(MAXW * 32, MAXW <= 4 ? 6 : 1) rmsnorm_quantize_kernel(
    const float* __restrict__ x, int64_t M, int64_t K, int64_t ldx, const float* __restrict__ gamma, float eps,
    const int32_t* __restrict__ rows, int64_t M_src, int64_t Mp, int8_t* __restrict__ q, float* __restrict__ scale,
    uint8_t* __restrict__ sums) {
    __shared__ double red[RMS_MAX_SB];
    __shared__ double rn_s;
    pdl_trigger();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int W = blockDim.x >> 5;
    const int64_t m = blockIdx.x;
    const int64_t nsb = K / QK;
    float xv[SBR][8];
    pdl_wait();  // x and rows may be outputs of the previous kernel on the stream
    int64_t src = m;
    if (rows != nullptr && m < M) {
        src = rows[m];
        if (src < 0 || src >= M_src) {
            if (threadIdx.x == 0) set_err(ERR_ROW_RANGE);
            src = -1;
        }
    }
    const bool live = m < M && src >= 0;
    const float* xr = x + (live ? src : 0) * ldx;
#pragma unroll
    for (int j = 0; j < SBR; j++) {
        const int64_t sj = w + (int64_t)j * W;
        if (sj < nsb && live) load8(xr + sj * QK + 8 * lane, xv[j]);
    }
    // one super-block per warp: its gamma too, so that pass 2 waits on no load
    float g1[8];
    if constexpr (SBR == 1) {
        if (w < nsb) load8(gamma + w * QK + 8 * lane, g1);
    }
#pragma unroll
    for (int j = 0; j < SBR; j++) {
        const int64_t sj = w + (int64_t)j * W;
        if (sj < nsb) {
            const double ps = butterfly_sum(live ? squares8(xv[j]) : 0.0);
            if (lane == 0) red[sj] = ps;
        }
    }
    for (int64_t sj = w + (int64_t)SBR * W; sj < nsb; sj += W) {
        float v[8];
        if (live) load8(xr + sj * QK + 8 * lane, v);
        const double ps = butterfly_sum(live ? squares8(v) : 0.0);
        if (lane == 0) red[sj] = ps;
    }
    __syncthreads();
    if (w == 0) {
        double t = lane < nsb ? red[lane] : 0.0;
        for (int64_t l = lane + 32; l < nsb; l += 32) t = __dadd_rn(t, red[l]);
        t = butterfly_sum(t);
        if (lane == 0) rn_s = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(t, (double)K), (double)eps)));
    }
    __syncthreads();
    const double rn = rn_s;
#pragma unroll
    for (int j = 0; j < SBR; j++) {
        const int64_t sj = w + (int64_t)j * W;
        if (sj < nsb) {
            float g8[8], v[8];
            if constexpr (SBR == 1) {
#pragma unroll
                for (int i = 0; i < 8; i++) g8[i] = g1[i];
            } else {
                load8(gamma + sj * QK + 8 * lane, g8);  // the same for every row: from L1
            }
#pragma unroll
            for (int i = 0; i < 8; i++)
                v[i] = live ? __double2float_rn(__dmul_rn(__dmul_rn((double)xv[j][i], rn), (double)g8[i])) : 0.0f;
            quantize_store_lane(v, lane, m, sj, Mp, q, scale, sums);
        }
    }
    for (int64_t sj = w + (int64_t)SBR * W; sj < nsb; sj += W) {
        float g8[8], x8[8], v[8];
        load8(gamma + sj * QK + 8 * lane, g8);
        if (live) load8(xr + sj * QK + 8 * lane, x8);
#pragma unroll
        for (int i = 0; i < 8; i++)
            v[i] = live ? __double2float_rn(__dmul_rn(__dmul_rn((double)x8[i], rn), (double)g8[i])) : 0.0f;
        quantize_store_lane(v, lane, m, sj, Mp, q, scale, sums);
    }
}

// The form of rmsnorm_quantize_kernel for Mp output rows of K on `sms` SMs: up to 12
// rows per SM, one super-block per warp and up to 32 warps (the shortest chain per row;
// with a partial wave, or behind the previous kernel's tail, the chain sets the time:
// at 512 and 1024 rows the wide form cost 3-5 us more per launch inside the step);
// beyond, up to 4 per warp and at most 4 warps, six CTAs per SM (rows in flight: 4096
// rows 46 -> 35 us).  Returns the warps per CTA; *wide tells which.
constexpr int RMS_WIDE_SBR = 4, RMS_WIDE_WARPS = 4;
inline int rms_warps(int64_t Mp, int64_t K, int sms, bool* wide) {
    const int64_t nsb = K / QK;
    *wide = Mp > 12 * (int64_t)sms;
    if (!*wide) return (int)(nsb < RMS_MAX_WARPS ? nsb : RMS_MAX_WARPS);
    const int64_t few = (nsb + RMS_WIDE_SBR - 1) / RMS_WIDE_SBR;
    return (int)(few < RMS_WIDE_WARPS ? few : RMS_WIDE_WARPS);
}

// SwiGLU + quantize.  Grid (Mp, ceil(nsb / 8)); warp w of CTA (m, b) handles
// super-block 8 b + w of canvas row m.  Rows M..Mp-1 are written as zeros.
__global__ void __launch_bounds__(FUSE_WARPS * 32) swiglu_quantize_kernel(
    const float* __restrict__ gate, const float* __restrict__ up, int64_t M, int64_t K, int64_t ld, int64_t Mp,
    int8_t* __restrict__ q, float* __restrict__ scale, uint8_t* __restrict__ sums) {
    pdl_trigger();
    pdl_wait();  // gate and up are normally the output of the previous kernel
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t m = blockIdx.x;
    const int64_t s = (int64_t)blockIdx.y * FUSE_WARPS + w;
    if (s >= K / QK) return;  // whole warp: no collective below spans warps
    float v[8];
    if (m < M) {
        float gv[8], uv[8];
        load8(gate + m * ld + s * QK + 8 * lane, gv);
        load8(up + m * ld + s * QK + 8 * lane, uv);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const double g = gv[i];
            const double silu = __ddiv_rn(g, __dadd_rn(1.0, exp(-g)));
            v[i] = __double2float_rn(__dmul_rn(silu, (double)uv[i]));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = 0.0f;
    }
    quantize_store_lane(v, lane, m, s, Mp, q, scale, sums);
}

}  // namespace dllm
