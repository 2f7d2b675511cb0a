// Device data layouts shared by the kernels of this library, the error word, and
// the load-time weight repack and activation quantization kernels.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dllm {

// ---------------------------------------------------------------- error word
// First device-detected error since the last dllm_get_device_status(); 0 = none.
__device__ int g_err;

__device__ __forceinline__ void set_err(int code) { atomicCAS(&g_err, 0, code); }

constexpr int ERR_ROW_RANGE = -5;
constexpr int ERR_TIMEOUT = -6;
constexpr int ERR_SCALE_RANGE = -9;

// ---------------------------------------------------------------- sizes
constexpr int QK = 256;             // weights per super-block
constexpr int TROWS = 128;          // weight rows per tile (= tensor-memory lanes)
constexpr int Q4K_BLOCK = 144;
constexpr int Q6K_BLOCK = 210;
constexpr int Q5K_BLOCK = 176;
constexpr int Q4K_TILE = TROWS * Q4K_BLOCK;  // 18432
constexpr int Q6K_TILE = TROWS * Q6K_BLOCK;  // 26880

// Q4_K tile: quants [8 pieces][128 rows][16 B] | scale bytes [128][12] | d,dmin [128][4]
constexpr int Q4K_OFF_SC = 8 * TROWS * 16;         // 16384
constexpr int Q4K_OFF_D = Q4K_OFF_SC + TROWS * 12;  // 17920
// Q6_K tile: low bits [8][128][16] | high bits [4][128][16] | scales [128][16] | d [128][2]
constexpr int Q6K_OFF_QH = 8 * TROWS * 16;          // 16384
constexpr int Q6K_OFF_SC = Q6K_OFF_QH + 4 * TROWS * 16;  // 24576
constexpr int Q6K_OFF_D = Q6K_OFF_SC + TROWS * 16;  // 26624

__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// ---------------------------------------------------------------- repack
// One thread per 16-byte chunk of the output.  Input blocks are read byte-wise
// (Q6_K blocks are 210 bytes and not 16-byte aligned).
__global__ void repack_q4k_kernel(const uint8_t* __restrict__ src, int64_t N, int64_t nsb,
                                  uint8_t* __restrict__ dst) {
    const int64_t chunks_per_tile = Q4K_TILE / 16;  // 1152
    const int64_t total = (N / TROWS) * nsb * chunks_per_tile;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = g / chunks_per_tile;
        const int c = (int)(g % chunks_per_tile);
        const int64_t t = tile / nsb, s = tile % nsb;
        uint8_t out[16];
        if (c < 1024) {  // quants: piece i of row r
            const int i = c / TROWS, r = c % TROWS;
            const uint8_t* blk = src + ((t * TROWS + r) * nsb + s) * Q4K_BLOCK;
#pragma unroll
            for (int b = 0; b < 16; b++) out[b] = blk[16 + 16 * i + b];
        } else if (c < 1024 + 96) {  // 12 scale bytes per row
            const int o = (c - 1024) * 16;
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int r = (o + b) / 12, j = (o + b) % 12;
                out[b] = src[((t * TROWS + r) * nsb + s) * Q4K_BLOCK + 4 + j];
            }
        } else {  // d, dmin: 4 bytes per row
            const int o = (c - 1120) * 16;
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int r = (o + b) / 4, j = (o + b) % 4;
                out[b] = src[((t * TROWS + r) * nsb + s) * Q4K_BLOCK + j];
            }
        }
        uint4 v;
        memcpy(&v, out, 16);
        reinterpret_cast<uint4*>(dst)[g] = v;
    }
}

// Q5_K (d, dmin, 12 scale bytes, 32 bytes of fifth bits qh, 128 bytes of low nibbles
// qs; weight d*sc_j*q - dmin*m_j with q = low nibble + 16 * fifth bit) as two Q4_K-form
// super-blocks of a matrix twice as wide: super-block s of a row becomes
//   s            the low nibbles: d, dmin, the same scale bytes, qs unchanged
//   nsb + s      the fifth bits as nibbles (0 or 1): d' = 16 d (exact: a power of two),
//                dmin' = 0, the same scale bytes
// so that d*sc*q - dmin*m = (d*sc*q4 - dmin*m) + (16 d)*sc*b exactly.  The result is in
// the Q4_K tile layout for nsb2 = 2 nsb super-blocks per row.
__global__ void repack_q5k_kernel(const uint8_t* __restrict__ src, int64_t N, int64_t nsb,
                                  uint8_t* __restrict__ dst) {
    const int64_t nsb2 = 2 * nsb;
    const int64_t chunks_per_tile = Q4K_TILE / 16;  // 1152
    const int64_t total = (N / TROWS) * nsb2 * chunks_per_tile;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = g / chunks_per_tile;
        const int c = (int)(g % chunks_per_tile);
        const int64_t t = tile / nsb2, s2 = tile % nsb2;
        const bool hi = s2 >= nsb;
        const int64_t s = hi ? s2 - nsb : s2;
        uint8_t out[16];
        if (c < 1024) {  // quants: piece i (bytes 16i..16i+15 of the 128) of row r
            const int i = c / TROWS, r = c % TROWS;
            const uint8_t* blk = src + ((t * TROWS + r) * nsb + s) * Q5K_BLOCK;
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int e = 16 * i + b, cc = e >> 5, l = e & 31;  // 32-byte chunk cc, element l
                const uint8_t qh = blk[16 + l];
                out[b] = hi ? (uint8_t)(((qh >> (2 * cc)) & 1) | (((qh >> (2 * cc + 1)) & 1) << 4)) : blk[48 + e];
            }
        } else if (c < 1024 + 96) {  // 12 scale bytes per row
            const int o = (c - 1024) * 16;
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int r = (o + b) / 12, j = (o + b) % 12;
                out[b] = src[((t * TROWS + r) * nsb + s) * Q5K_BLOCK + 4 + j];
            }
        } else {  // d, dmin: 4 bytes per row
            const int o = (c - 1120) * 16;
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int r = (o + b) / 4, j = (o + b) % 4;
                const uint8_t* blk = src + ((t * TROWS + r) * nsb + s) * Q5K_BLOCK;
                if (!hi) {
                    out[b] = blk[j];
                } else if (j < 2) {
                    // 16 d is exact in f16 unless it overflows: |d| >= 4096 cannot be split
                    const unsigned short dbits = (unsigned short)(blk[0] | (blk[1] << 8));
                    const float d16f = 16.0f * __half2float(__ushort_as_half(dbits));
                    if (j == 0 && !(fabsf(d16f) <= 65504.0f)) set_err(ERR_SCALE_RANGE);
                    const unsigned short d16 = __half_as_ushort(__float2half_rn(d16f));
                    out[b] = (uint8_t)(j == 0 ? d16 & 255 : d16 >> 8);
                } else {
                    out[b] = 0;  // dmin' = +0
                }
            }
        }
        uint4 v;
        memcpy(&v, out, 16);
        reinterpret_cast<uint4*>(dst)[g] = v;
    }
}

__global__ void repack_q6k_kernel(const uint8_t* __restrict__ src, int64_t N, int64_t nsb,
                                  uint8_t* __restrict__ dst) {
    const int64_t chunks_per_tile = Q6K_TILE / 16;  // 1680
    const int64_t total = (N / TROWS) * nsb * chunks_per_tile;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = g / chunks_per_tile;
        const int c = (int)(g % chunks_per_tile);
        const int64_t t = tile / nsb, s = tile % nsb;
        uint8_t out[16];
        if (c < 1536) {  // low bits (pieces 0..7) then high bits (pieces 8..11), 16 B per row
            const int i = c / TROWS, r = c % TROWS;
            const uint8_t* blk = src + ((t * TROWS + r) * nsb + s) * Q6K_BLOCK;
#pragma unroll
            for (int b = 0; b < 16; b++) out[b] = blk[16 * i + b];
        } else if (c < 1664) {  // 16 int8 scales per row
            const int r = c - 1536;
            const uint8_t* blk = src + ((t * TROWS + r) * nsb + s) * Q6K_BLOCK;
#pragma unroll
            for (int b = 0; b < 16; b++) out[b] = blk[192 + b];
        } else {  // d: 2 bytes per row
            const int o = (c - 1664) * 16;
#pragma unroll
            for (int b = 0; b < 16; b++) {
                const int r = (o + b) / 2, j = (o + b) % 2;
                out[b] = src[((t * TROWS + r) * nsb + s) * Q6K_BLOCK + 208 + j];
            }
        }
        uint4 v;
        memcpy(&v, out, 16);
        reinterpret_cast<uint4*>(dst)[g] = v;
    }
}

// ---------------------------------------------------------------- quantize_act
// One CTA of 8 warps per (8-row group g, super-block s); warp w owns row 8g + w.
// Lane l holds elements 8l..8l+7 of the 256-block: amax by warp reduction, then
// iscale = 127/amax and scale = amax/127 as IEEE f32 divisions, qa =
// round-half-even(x * iscale) clamped to [-127, 127].  For each sub-block of 32 the
// sum t_j of its qa values is also emitted multiplied by the block scale, as two
// floats v_hi + v_lo = scale * t_j (v_hi exact as a tf32 operand): the B operand of
// the min-term MMA of Q4_K weights.  Outputs are staged in shared memory in the
// tensor-core operand order and written with 16-byte stores.
__global__ void __launch_bounds__(256) quantize_act_kernel(const float* __restrict__ x, int64_t M, int64_t ldx,
                                                           int64_t Mp, int8_t* __restrict__ q,
                                                           float* __restrict__ scale,
                                                           uint8_t* __restrict__ sums) {
    __shared__ __align__(16) uint8_t tile[16 * 8 * 16];  // [chunk][row][16 B]
    __shared__ __align__(16) float tsum[4 * 8 * 4];      // [hi j0-3, hi j4-7, lo j0-3, lo j4-7][row][4]
    __shared__ float tscale[8];
    pdl_trigger();
    pdl_wait();  // x may be the output of the previous kernel on the stream
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t g = blockIdx.x, s = blockIdx.y;
    const int64_t m = 8 * g + w;
    float v[8];
    if (m < M) {
        const float4* p = reinterpret_cast<const float4*>(x + m * ldx + s * QK + 8 * lane);
        const float4 a = __ldg(p), b = __ldg(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = 0.0f;
    }
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
    // lane l -> chunk l/2, half l%2 of row w
    *reinterpret_cast<uint2*>(&tile[((lane >> 1) * 8 + w) * 16 + (lane & 1) * 8]) = make_uint2(packed[0], packed[1]);
    // sub-block j (32 elements) is held by lanes 4j..4j+3
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if ((lane & 3) == 0) {
        const int j = lane >> 2;
        float hi, lo;
        split_tf32(__fmul_rn(sc, (float)part), hi, lo);
        tsum[((j >> 2) * 8 + w) * 4 + (j & 3)] = hi;
        tsum[((2 + (j >> 2)) * 8 + w) * 4 + (j & 3)] = lo;
    }
    if (lane == 0) tscale[w] = sc;
    __syncthreads();
    const int tid = threadIdx.x;
    if (tid < 128) {
        uint4* dq = reinterpret_cast<uint4*>(q + ((s * (Mp / 8) + g) * 16) * 128);
        dq[tid] = reinterpret_cast<const uint4*>(tile)[tid];
    } else if (tid < 160) {
        uint4* ds = reinterpret_cast<uint4*>(sums + (s * (Mp / 8) + g) * 512);
        ds[tid - 128] = reinterpret_cast<const uint4*>(tsum)[tid - 128];
    } else if (tid < 168) {
        scale[s * Mp + 8 * g + (tid - 160)] = tscale[tid - 160];
    }
}

}  // namespace dllm
