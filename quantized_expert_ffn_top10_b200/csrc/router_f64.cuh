// Router logits of a short chunk (MOE_DECODE_MAX_T < T <= MOE_ROUTER_F64_MAX_T)
// in fp64 on the tensor cores (mma.m8n8k4.f64), for the certified top-k of
// the "Strata Coder deep-dive" page, section 1 (10 of 512 experts per token).
//
// A chunk this short gives the bf16-plane tensor-core router of long chunks
// only E / 128 tiles to run, each a full pass over H on one SM.  Here a CTA
// takes 8 experts (the MMA's A rows) x 8 tokens (its B columns) and its 16
// warps split H, so the work spreads over (E / 8) x (T / 8) CTAs.  Every
// bf16 x fp32 product is exact in fp64 and only the additions round: along
// any product's path at most H + 32 of them (the per-warp MMA chains, the two
// half-slice chains, the cross-warp sum and the bias), which the top-k's
// bound gamma_(H+32) (||x|| ||W_r[e]|| + |b_e|) covers.
#pragma once
#include "common.cuh"

#define RF_WARPS 16

// logit [T][E] fp64; wnorm [E] (written by the CTAs of the first token group):
// ||W_r[e]||_2 inflated over its fp32 rounding.  Needs H % 32 == 0 and
// 16-byte aligned W_r rows and x rows.
__global__ void __launch_bounds__(32 * RF_WARPS)
    k_router_f64(const uint16_t* __restrict__ x, int T, int H, const float* __restrict__ W,
                 const float* __restrict__ b, int E, double* __restrict__ logit, float* __restrict__ wnorm) {
    __shared__ double s_part[RF_WARPS][8][8];  // [warp][expert][token]
    __shared__ float s_w2[RF_WARPS][8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int e0 = blockIdx.x * 8, t0 = blockIdx.y * 8;
    const bool erow = e0 + g < E, xrow = t0 + g < T;
    const float* wr = W + (size_t)(erow ? e0 + g : 0) * H;
    const uint16_t* xr = x + (size_t)(xrow ? t0 + g : 0) * H;
    // A element (row g, column q) of MMA step st is W_r[e0 + g][k1 + 4 q + st], B element
    // (row q, column g) is x[t0 + g][k1 + 4 q + st]: the same k on both sides
    double c0 = 0.0, c1 = 0.0, d0 = 0.0, d1 = 0.0;  // two chains: the even and the odd 16-element half
    float w2 = 0.f;
#pragma unroll 2
    for (int k0 = warp * 32; k0 < H; k0 += 32 * RF_WARPS) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int k1 = k0 + 16 * half + 4 * q;
            const float4 wv = erow ? __ldg(reinterpret_cast<const float4*>(wr + k1)) : make_float4(0.f, 0.f, 0.f, 0.f);
            const uint2 xv = xrow ? __ldg(reinterpret_cast<const uint2*>(xr + k1)) : make_uint2(0u, 0u);
            w2 = fmaf(wv.x, wv.x, fmaf(wv.y, wv.y, fmaf(wv.z, wv.z, fmaf(wv.w, wv.w, w2))));
            const double av[4] = {wv.x, wv.y, wv.z, wv.w};
            const double bv[4] = {__uint_as_float(xv.x << 16), __uint_as_float(xv.x & 0xffff0000u),
                                  __uint_as_float(xv.y << 16), __uint_as_float(xv.y & 0xffff0000u)};
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                if (half == 0)
                    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                                 : "+d"(c0), "+d"(c1)
                                 : "d"(av[st]), "d"(bv[st]));
                else
                    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                                 : "+d"(d0), "+d"(d1)
                                 : "d"(av[st]), "d"(bv[st]));
            }
        }
    }
    // D element (row g, columns 2q, 2q + 1): expert e0 + g, tokens t0 + 2q, t0 + 2q + 1
    s_part[warp][g][2 * q] = c0 + d0;
    s_part[warp][g][2 * q + 1] = c1 + d1;
    w2 += __shfl_xor_sync(0xffffffffu, w2, 1);
    w2 += __shfl_xor_sync(0xffffffffu, w2, 2);
    if (q == 0) s_w2[warp][g] = w2;
    __syncthreads();
    if (threadIdx.x < 64) {
        const int gg = threadIdx.x >> 3, n = threadIdx.x & 7, e = e0 + gg, t = t0 + n;
        if (e < E && t < T) {
            double p4[4] = {0.0, 0.0, 0.0, 0.0};  // four short chains over the warps, in a fixed order
#pragma unroll
            for (int w = 0; w < RF_WARPS; ++w) p4[w & 3] += s_part[w][gg][n];
            double s = (p4[0] + p4[1]) + (p4[2] + p4[3]);
            if (b) s += (double)b[e];
            logit[(size_t)t * E + e] = s;
        }
    } else if (blockIdx.y == 0 && threadIdx.x < 72) {
        const int gg = threadIdx.x - 64, e = e0 + gg;
        if (e < E) {
            float s2 = 0.f;
#pragma unroll
            for (int w = 0; w < RF_WARPS; ++w) s2 += s_w2[w][gg];
            wnorm[e] = sqrtf(s2) * 1.001f;
        }
    }
}
