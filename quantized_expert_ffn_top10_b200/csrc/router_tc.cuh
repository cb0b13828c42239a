// Router logits of a prefill chunk on the 5th-generation tensor cores.
//
// W_r (fp32) is split exactly into three bf16 planes, w = hi + mid + lo (each
// step keeps 8 of the 24 significand bits; bf16 has fp32's exponent range), so
// every product x * plane (bf16 x bf16) is exact in fp32 and
//     logit[t][e] = sum_h x[t][h] (hi + mid + lo)[e][h] + b[e]
// is one fp32-accumulated contraction of K = 3H exact terms.  The certified
// top-k bounds its rounding (see moe_tc_router_gamma) and re-evaluates close
// calls in fp64, so the selection is the definition's.
//
// k_router_split: planes [3][E][H] bf16 and row norms (upper bounds of ||W[e]||).
// k_router_tc: a tile is 128 experts (M, the weight rows) x 128 tokens (N);
// warp 0 issues TMA loads of the three plane tiles and the token tile
// (128-byte swizzled, K-major), warp 1 owns TMEM and issues tcgen05.mma,
// warps 2-5 move the fp32 accumulators to the logits (+ bias).  Three TMEM
// accumulators keep the rounding small: the hi plane over the first and the
// second half of K, and the mid and lo planes (2^-8 and 2^-16 of the weight)
// together; the epilogue adds them in a fixed order.
#pragma once
#include "common.cuh"

#define RT_BM 128      // experts per tile
#define RT_BN 128      // tokens per tile
#define RT_BK 64       // K per stage (one 128-byte swizzle row of bf16)
#define RT_STAGES 3
#define RT_THREADS 192
#define RT_TILE_BYTES (128 * RT_BK * 2)                  // 16 KB: 128 rows x 128 B
#define RT_STAGE_BYTES (4 * RT_TILE_BYTES)               // three planes + tokens
#define RT_SMEM (RT_STAGES * RT_STAGE_BYTES + 1024 + 256)

// Planes and row norms.  One CTA per expert row; thread i takes elements i, i + 256, ...
__global__ void __launch_bounds__(256) k_router_split(const float* __restrict__ W, int E, int H,
                                                      uint16_t* __restrict__ planes, float* __restrict__ wnorm) {
    const int e = blockIdx.x;
    __shared__ float s_red[8];
    float ss = 0.f;
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        const float w = W[(size_t)e * H + h];
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(hi);  // exact
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);  // exact, at most 8 significant bits
        const __nv_bfloat16 lo = __float2bfloat16_rn(r2);  // exact
        planes[(size_t)e * H + h] = __bfloat16_as_ushort(hi);
        planes[((size_t)E + e) * H + h] = __bfloat16_as_ushort(mid);
        planes[((size_t)2 * E + e) * H + h] = __bfloat16_as_ushort(lo);
        ss = fmaf(w, w, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += s_red[i];
        wnorm[e] = sqrtf(t) * 1.001f;  // inflated over its own fp32 rounding
    }
}

// grid (E / RT_BM, ceil(T / RT_BN)); tmA: planes as [3E][H] bf16, box 64 x 128;
// tmB: x as [T][H] bf16, box 64 x 128 (rows past T read as zero).
__global__ void __launch_bounds__(RT_THREADS, 1)
    k_router_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int T, int H, int E,
                const float* __restrict__ b, float* __restrict__ logit) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + RT_STAGES * RT_STAGE_BYTES);
    uint64_t* empty = full + RT_STAGES;
    uint64_t* accf = empty + RT_STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * RT_BM, n0 = blockIdx.y * RT_BN, nk = H / RT_BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RT_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 4 * RT_BN);  // three accumulators of RT_BN columns (a power of two is allocated)
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % RT_STAGES, ph = (kb / RT_STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, 21, kb)) break;
                uint8_t* st = smem + s * RT_STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], RT_STAGE_BYTES);
#pragma unroll
                for (int p = 0; p < 3; ++p) tma_load_2d(st + p * RT_TILE_BYTES, &tmA, &full[s], kb * RT_BK, p * E + m0);
                tma_load_2d(st + 3 * RT_TILE_BYTES, &tmB, &full[s], kb * RT_BK, n0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(RT_BM, RT_BN);
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % RT_STAGES, ph = (kb / RT_STAGES) & 1;
                ok = mbar_wait(&full[s], ph, 22, kb);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * RT_STAGE_BYTES);
                const bool first_half = kb < nk / 2;
#pragma unroll
                for (int kk = 0; kk < RT_BK / 16; ++kk) {
                    const uint64_t bdesc = make_sdesc_sw128(st + 3 * RT_TILE_BYTES + kk * 32);
                    // hi plane -> accumulator 0 (first half of K) or 1 (second half)
                    tc_mma_bf16(tmem + (first_half ? 0 : RT_BN), make_sdesc_sw128(st + kk * 32), bdesc, idesc,
                                (kb != 0 && kb != nk / 2) || kk != 0);
                    // mid and lo planes -> accumulator 2
#pragma unroll
                    for (int p = 1; p < 3; ++p)
                        tc_mma_bf16(tmem + 2 * RT_BN, make_sdesc_sw128(st + p * RT_TILE_BYTES + kk * 32), bdesc, idesc,
                                    (kb | kk) != 0 || p != 1);
                }
                tc_commit(&empty[s]);
            }
            tc_commit(accf);  // arrives once every MMA issued above has completed
        }
    } else {  // warps 2..5: TMEM lane quadrant warp % 4 holds experts m0 + 32 (warp % 4) + lane
        const int q = warp & 3, e = m0 + q * 32 + lane;
        const bool okw = mbar_wait(accf, 0, 23, 0);
        tc_fence_after();
        const float be = (b && okw) ? b[e] : 0.f;
        const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16);
        for (int c0 = 0; c0 < RT_BN && okw; c0 += 16) {
            uint32_t v0[16], v1[16], v2[16];
            tmem_ld16(ta + c0, v0);
            tmem_ld16(ta + RT_BN + c0, v1);
            tmem_ld16(ta + 2 * RT_BN + c0, v2);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int t = n0 + c0 + j;
                const float lg = (__uint_as_float(v0[j]) + __uint_as_float(v1[j])) + __uint_as_float(v2[j]);
                if (t < T) logit[(size_t)t * E + e] = lg + be;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 4 * RT_BN);
}

// Bound factor of the tensor-core logits: |computed - exact| <= gamma * sum |x w|
// (and sum |x w| <= ||x|| ||w||).  The model: every MMA step adds a 16-term
// partial sum of exact products to its fp32 accumulator; the partial sum may
// carry an error of 2^-20 of its terms (a truncating adder) and the addition
// one rounding (2^-23, truncation-safe) of the running sum, which is bounded by
// the sum of |terms| so far.  Accumulators 0 and 1 (hi plane, one half of K
// each) take H/32 steps, accumulator 2 (mid + lo, at most 2^-8 (1 + 2^-8) of
// |w|) takes H/8 steps, and the epilogue adds three times.  |hi| <= |w| (1 +
// 2^-8).  The total is doubled as a margin for the unknown adder.
__host__ __device__ inline double moe_tc_router_gamma(int H) {
    const double u = 1.1920928955078125e-07, part = 9.5367431640625e-07;  // 2^-23, 2^-20
    const double g_hi = (H / 32.0 + 3.0) * u + part;
    const double g_ml = ((H / 8.0) * u + part) * (1.0 / 256.0) * (1.0 + 1.0 / 256.0);
    return 2.0 * (g_hi + g_ml) * (1.0 + 1.0 / 256.0);
}
