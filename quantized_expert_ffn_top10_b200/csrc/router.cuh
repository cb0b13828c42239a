// Router: logits l[t][e] = x_t . W_r[e] + b_e, top-k selection that is
// bit-exact against the fp64 definition, and the softmax gate weights.
//
// Selection is certified.  The fast logits (fp32) carry a rigorous error
// bound delta_e = gamma_n * B_e, where n is the longest chain of roundings in
// their summation and B_e >= sum_h |x_h W_eh| + |b_e|.  The best k+2 candidates
// are re-evaluated in fp64 (again with a bound).  When every gap that decides
// the selection or the order of the k chosen experts exceeds the combined
// bounds, the result equals the fp64 definition summed in index order.
// Otherwise the token is re-evaluated exactly: every expert that could still
// reach the top k gets its logit summed sequentially over h in fp64, which is
// the definition itself (each bf16 x fp32 product is exact in fp64, so the
// fused multiply-add sequence reproduces it bit for bit), and the selection is
// taken on those values with ties going to the lower expert index.
#pragma once
#include "common.cuh"

#define MOE_TOPK_WARPS 4
#define MOE_CAND_EXTRA 2  // fp64 candidates beyond k

// ---------------------------------------------------------------- column max for the prefill bound

// cmax[h] = max_e |W[e][h]| (h < H), cmax[H] = max_e |b_e|, as float bits.
// The caller zeroes cmax first; all values are >= 0 so unsigned max is exact.
__global__ void k_router_colmax(const float* __restrict__ W, const float* __restrict__ b, int E, int H,
                                unsigned int* __restrict__ cmax) {
    int h = blockIdx.x * blockDim.x + threadIdx.x;
    int e0 = blockIdx.y * 32, e1 = min(E, e0 + 32);
    if (h < H) {
        float m = 0.f;
        for (int e = e0; e < e1; ++e) m = fmaxf(m, fabsf(__ldg(W + (size_t)e * H + h)));
        atomicMax(cmax + h, __float_as_uint(m));
    } else if (h == H && b != nullptr) {
        float m = 0.f;
        for (int e = e0; e < e1; ++e) m = fmaxf(m, fabsf(b[e]));
        atomicMax(cmax + H, __float_as_uint(m));
    }
}

// ---------------------------------------------------------------- decode router: GEMV, warp per expert

// Fast logits and per-entry bounds for T <= MOE_DECODE_MAX_T tokens.  Lane L
// sums h = 4L + 128i + j sequentially (chain H/32), then a 5-level butterfly
// and the bias: chain length H/32 + 6.  absum[t][e] = sum |x W| + |b|.
__global__ void __launch_bounds__(256) k_router_gemv(const uint16_t* __restrict__ x, int T, int H,
                                                     const float* __restrict__ W, const float* __restrict__ b,
                                                     int E, float* __restrict__ logit, float* __restrict__ absum) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= E) return;
    float acc[MOE_DECODE_MAX_T], ab[MOE_DECODE_MAX_T];
#pragma unroll
    for (int t = 0; t < MOE_DECODE_MAX_T; ++t) acc[t] = ab[t] = 0.f;
    const float4* w4 = reinterpret_cast<const float4*>(W + (size_t)e * H);
    for (int i = lane; i < H / 4; i += 32) {
        float4 w = __ldg(w4 + i);
#pragma unroll
        for (int t = 0; t < MOE_DECODE_MAX_T; ++t) {
            if (t < T) {
                uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + (size_t)t * H) + i);
                float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
                float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
                acc[t] = fmaf(x0, w.x, acc[t]);
                acc[t] = fmaf(x1, w.y, acc[t]);
                acc[t] = fmaf(x2, w.z, acc[t]);
                acc[t] = fmaf(x3, w.w, acc[t]);
                ab[t] = fmaf(fabsf(x0), fabsf(w.x), ab[t]);
                ab[t] = fmaf(fabsf(x1), fabsf(w.y), ab[t]);
                ab[t] = fmaf(fabsf(x2), fabsf(w.z), ab[t]);
                ab[t] = fmaf(fabsf(x3), fabsf(w.w), ab[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < MOE_DECODE_MAX_T; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
            ab[t] += __shfl_xor_sync(0xffffffffu, ab[t], o);
        }
    }
    if (lane == 0) {
        float bb = b ? b[e] : 0.f;
        for (int t = 0; t < T; ++t) {
            logit[(size_t)t * E + e] = acc[t] + bb;
            absum[(size_t)t * E + e] = ab[t] + fabsf(bb);
        }
    }
}

// ---------------------------------------------------------------- prefill router: fp32 tiled GEMM

#define RG_BM 128
#define RG_BN 64
#define RG_BK 16

// l[t][e] = sum_h x[t][h] W[e][h] + b_e, each output summed sequentially over
// h by one thread (chain length H + 1).
__global__ void __launch_bounds__(256) k_router_gemm(const uint16_t* __restrict__ x, int T, int H,
                                                     const float* __restrict__ W, const float* __restrict__ b,
                                                     int E, float* __restrict__ logit) {
    __shared__ __align__(16) float Xs[RG_BK][RG_BM + 4];
    __shared__ __align__(16) float Ws[RG_BK][RG_BN + 4];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int t0 = blockIdx.y * RG_BM, e0 = blockIdx.x * RG_BN;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    // loader assignment: X: row tid/2, k (tid%2)*8 (8 bf16); W: row tid/4, k (tid%4)*4 (4 fp32)
    const int xr = tid >> 1, xk = (tid & 1) * 8;
    const int wr = tid >> 2, wk = (tid & 3) * 4;
    const bool xok = (t0 + xr) < T, wok = (e0 + wr) < E;
    const uint16_t* xp = x + (size_t)(t0 + xr) * H + xk;
    const float* wp = W + (size_t)(e0 + wr) * H + wk;
    uint4 xa = xok ? __ldg(reinterpret_cast<const uint4*>(xp)) : make_uint4(0, 0, 0, 0);
    float4 wa = wok ? __ldg(reinterpret_cast<const float4*>(wp)) : make_float4(0, 0, 0, 0);
    for (int k0 = 0; k0 < H; k0 += RG_BK) {
        __syncthreads();
        Xs[xk + 0][xr] = __uint_as_float(xa.x << 16);
        Xs[xk + 1][xr] = __uint_as_float(xa.x & 0xffff0000u);
        Xs[xk + 2][xr] = __uint_as_float(xa.y << 16);
        Xs[xk + 3][xr] = __uint_as_float(xa.y & 0xffff0000u);
        Xs[xk + 4][xr] = __uint_as_float(xa.z << 16);
        Xs[xk + 5][xr] = __uint_as_float(xa.z & 0xffff0000u);
        Xs[xk + 6][xr] = __uint_as_float(xa.w << 16);
        Xs[xk + 7][xr] = __uint_as_float(xa.w & 0xffff0000u);
        Ws[wk + 0][wr] = wa.x;
        Ws[wk + 1][wr] = wa.y;
        Ws[wk + 2][wr] = wa.z;
        Ws[wk + 3][wr] = wa.w;
        __syncthreads();
        if (k0 + RG_BK < H) {  // prefetch the next tile while computing this one
            xa = xok ? __ldg(reinterpret_cast<const uint4*>(xp + k0 + RG_BK)) : make_uint4(0, 0, 0, 0);
            wa = wok ? __ldg(reinterpret_cast<const float4*>(wp + k0 + RG_BK)) : make_float4(0, 0, 0, 0);
        }
#pragma unroll
        for (int kk = 0; kk < RG_BK; ++kk) {
            float4 a0 = *reinterpret_cast<const float4*>(&Xs[kk][ty * 8]);
            float4 a1 = *reinterpret_cast<const float4*>(&Xs[kk][ty * 8 + 4]);
            float4 bv = *reinterpret_cast<const float4*>(&Ws[kk][tx * 4]);
            float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int t = t0 + ty * 8 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int e = e0 + tx * 4 + j;
            if (e < E) logit[(size_t)t * E + e] = acc[i][j] + (b ? b[e] : 0.f);
        }
    }
}

// ---------------------------------------------------------------- certified top-k

struct TopkArgs {
    const uint16_t* x;       // [T][H] bf16
    const float* W;          // [E][H]
    const float* b;          // [E] or null
    const float* logit;      // [T][E] fast fp32 logits
    const float* absum;      // [T][E] per-entry bound sums, or null -> use cmax
    const unsigned int* cmax;  // [H+1] column maxima (float bits), used when absum == null
    int32_t* idx;            // [T][k]
    float* w;                // [T][k]
    int32_t* n_rechecked;    // [1] or null
    float gamma32;           // bound factor of the fast logits: n u / (1 - n u)
    int T, H, E, k;
};

// warp-wide argmax of (v desc, e asc); every lane returns the winner
__device__ __forceinline__ void warp_best(float& v, int& e) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        int e2 = __shfl_xor_sync(0xffffffffu, e, o);
        if (v2 > v || (v2 == v && e2 < e)) { v = v2; e = e2; }
    }
}

__device__ __forceinline__ void warp_best_d(double& v, int& e) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        double v2 = __shfl_xor_sync(0xffffffffu, v, o);
        int e2 = __shfl_xor_sync(0xffffffffu, e, o);
        if (v2 > v || (v2 == v && e2 < e)) { v = v2; e = e2; }
    }
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// fp64 logit of expert e for token t, summed over lane-strided chains of
// length H/32 and a 5-level butterfly; also returns sum |x W| + |b|.
__device__ __forceinline__ void logit_fp64_parallel(const TopkArgs& a, int t, int e, double& v, double& ab) {
    const int lane = threadIdx.x & 31;
    const uint16_t* xr = a.x + (size_t)t * a.H;
    const float* wr = a.W + (size_t)e * a.H;
    double s = 0.0, sa = 0.0;
    for (int h = lane; h < a.H; h += 32) {
        double p = (double)bf16_bits_to_f32(xr[h]) * (double)__ldg(wr + h);
        s += p;
        sa += fabs(p);
    }
    s = warp_sum_d(s);
    sa = warp_sum_d(sa);
    double bb = a.b ? (double)a.b[e] : 0.0;
    v = s + bb;
    ab = sa + fabs(bb);
}

// The definition: fp64, sequential over h, then + b.  One thread.
__device__ __forceinline__ double logit_fp64_exact(const TopkArgs& a, int t, int e) {
    const uint16_t* xr = a.x + (size_t)t * a.H;
    const float* wr = a.W + (size_t)e * a.H;
    double s = 0.0;
    for (int h = 0; h < a.H; ++h) s = fma((double)bf16_bits_to_f32(xr[h]), (double)__ldg(wr + h), s);
    if (a.b) s += (double)a.b[e];
    return s;
}

// One warp per token.  Lanes hold logits of experts e = lane + 32 i.
__global__ void __launch_bounds__(32 * MOE_TOPK_WARPS) k_topk(TopkArgs a) {
    __shared__ int s_ce[MOE_TOPK_WARPS][MOE_MAX_E];
    __shared__ double s_cv[MOE_TOPK_WARPS][MOE_MAX_E];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t = blockIdx.x * MOE_TOPK_WARPS + wid;
    if (t >= a.T) return;
    const int E = a.E, k = a.k, H = a.H;
    constexpr int NV = MOE_MAX_E / 32;
    const double u64 = 1.1102230246251565e-16;  // 2^-53
    // oracle's own rounding bound (sequential fp64, chain H + 1) per unit of B
    const double g_or = (double)(H + 2) * u64 * 1.01;

    // per-token bound when no per-entry sums exist: B = sum_h |x_h| cmax_h + max|b|
    float Btok = 0.f;
    if (!a.absum) {
        const uint16_t* xr = a.x + (size_t)t * H;
        float s = 0.f;
        for (int h = lane; h < H; h += 32) s = fmaf(fabsf(bf16_bits_to_f32(xr[h])), __uint_as_float(a.cmax[h]), s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        // this fp32 sum of nonnegative terms (chain H/32 + 5) can be low by a
        // relative 2 gamma at most; 1% covers it for any H here
        Btok = s * 1.01f + (a.b ? __uint_as_float(a.cmax[H]) : 0.f) * 1.01f;
    }
    float v[NV], dl[NV];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        int e = lane + 32 * i;
        if (e < E) {
            v[i] = a.logit[(size_t)t * E + e];
            float B = a.absum ? a.absum[(size_t)t * E + e] * 1.01f : Btok;
            dl[i] = B * (a.gamma32 * 1.01f) + (float)(B * g_or) + 1e-30f;
        } else {
            v[i] = -INFINITY;
            dl[i] = 0.f;
            taken |= 1u << i;
        }
    }
    // 1) top M by the fast logits
    const int M = min(min(E, k + MOE_CAND_EXTRA), 32);
    int my_e = -1;  // lane j < M holds candidate j
    for (int j = 0; j < M; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NV; ++i)
            if (!(taken >> i & 1u)) {
                int e = lane + 32 * i;
                if (v[i] > bv || (v[i] == bv && e < be)) { bv = v[i]; be = e; }
            }
        warp_best(bv, be);
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) my_e = be;
    }
    // upper end of every expert outside the candidates
    float rest = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV; ++i)
        if (!(taken >> i & 1u)) rest = fmaxf(rest, v[i] + dl[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rest = fmaxf(rest, __shfl_xor_sync(0xffffffffu, rest, o));

    // 2) fp64 re-evaluation of the candidates (warp-parallel, bounded)
    const double g_par = (double)(H / 32 + 8) * u64 * 1.01;
    double cv = -INFINITY, cd = 0.0;
    for (int j = 0; j < M; ++j) {
        int e = __shfl_sync(0xffffffffu, my_e, j);
        double vv, ab;
        logit_fp64_parallel(a, t, e, vv, ab);
        if (lane == j) { cv = vv; cd = ab * (g_par + g_or) + 1e-300; }
    }
    // 3) sorted position of each candidate by (cv desc, e asc)
    int rank = 0;
    for (int j = 0; j < M; ++j) {
        double oj = __shfl_sync(0xffffffffu, cv, j);
        int ej = __shfl_sync(0xffffffffu, my_e, j);
        if (lane < M && (oj > cv || (oj == cv && ej < my_e))) ++rank;
    }
    // gather candidates into sorted order: lane r receives position r
    int src = 0;
    for (int j = 0; j < M; ++j) {
        int rj = __shfl_sync(0xffffffffu, rank, j);
        if (rj == lane) src = j;
    }
    double sv = __shfl_sync(0xffffffffu, cv, src);
    double sd = __shfl_sync(0xffffffffu, cd, src);
    int se = __shfl_sync(0xffffffffu, my_e, src);
    double nv = __shfl_down_sync(0xffffffffu, sv, 1);
    double nd = __shfl_down_sync(0xffffffffu, sd, 1);
    // 4) certification: positions r < k are strictly separated from r + 1
    //    (when it exists) and the k-th chosen clears every non-candidate
    bool ok = true;
    if (lane < k && lane + 1 < M) ok = (sv - sd) > (nv + nd);
    if (lane == k - 1) ok = ok && ((sv - sd) > (double)rest || rest == -INFINITY);
    const bool certified = __all_sync(0xffffffffu, ok);

    if (certified) {
        double v0 = __shfl_sync(0xffffffffu, sv, 0);
        double z = (lane < k) ? exp(sv - v0) : 0.0;
        double zs = warp_sum_d(z);
        if (lane < k) {
            a.idx[(size_t)t * k + lane] = se;
            a.w[(size_t)t * k + lane] = (float)(z / zs);
        }
        return;
    }

    // 5) exact path: every expert whose upper end reaches theta, the lowest
    //    lower end among the chosen k, is evaluated by the definition
    double th = (lane < k) ? (sv - sd) : INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) th = fmin(th, __shfl_xor_sync(0xffffffffu, th, o));
    int* ce = s_ce[wid];
    double* cvs = s_cv[wid];
    int nc = 0;
    for (int i = 0; i < NV; ++i) {
        int e = lane + 32 * i;
        // the candidates of step 1 (marked taken) are always kept
        bool in = (e < E) && (((taken >> i) & 1u) || (double)v[i] + (double)dl[i] >= th);
        unsigned m = __ballot_sync(0xffffffffu, in);
        if (in) ce[nc + __popc(m & ((1u << lane) - 1))] = e;
        nc += __popc(m);
    }
    __syncwarp();
    for (int c = lane; c < nc; c += 32) cvs[c] = logit_fp64_exact(a, t, ce[c]);
    __syncwarp();
    // select k from the exact values, ties to the lower index
    double l0 = 0.0, z = 0.0;
    for (int j = 0; j < k; ++j) {
        double bv = -INFINITY;
        int be = 0x7fffffff, bc = -1;
        for (int c = lane; c < nc; c += 32)
            if (ce[c] >= 0 && (cvs[c] > bv || (cvs[c] == bv && ce[c] < be))) { bv = cvs[c]; be = ce[c]; bc = c; }
        int bcw = bc;
        double bvw = bv;
        int bew = be;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            double v2 = __shfl_xor_sync(0xffffffffu, bvw, o);
            int e2 = __shfl_xor_sync(0xffffffffu, bew, o);
            int c2 = __shfl_xor_sync(0xffffffffu, bcw, o);
            if (v2 > bvw || (v2 == bvw && e2 < bew)) { bvw = v2; bew = e2; bcw = c2; }
        }
        __syncwarp();
        if (lane == 0) {
            ce[bcw] = -1;  // remove from the pool
            a.idx[(size_t)t * k + j] = bew;
        }
        __syncwarp();
        if (j == 0) l0 = bvw;
        double zz = exp(bvw - l0);
        z += zz;
        if (lane == j) cd = zz;  // reuse: lane j keeps its numerator
    }
    if (lane < k) a.w[(size_t)t * k + lane] = (float)(cd / z);
    if (lane == 0 && a.n_rechecked) atomicAdd(a.n_rechecked, 1);
}
