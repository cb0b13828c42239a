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
#include <type_traits>

#include "common.cuh"

#define MOE_TOPK_WARPS 4
#define MOE_CAND_EXTRA 2  // fp64 candidates beyond k

// ---------------------------------------------------------------- decode router: fp64 GEMV, warp per expert

// Logits in fp64 for T <= MOE_DECODE_MAX_T tokens, with per-entry bound sums.
// Lane L sums h = 4L + 128i + j sequentially (chain H/32), then a 5-level
// butterfly and the bias: chain length H/32 + 6.  absum[t][e] = sum |x W| + |b|.
// fp64 costs nothing here: the kernel is bound by reading W (4 B per weight).
__global__ void __launch_bounds__(256) k_router_gemv(const uint16_t* __restrict__ x, int T, int H,
                                                     const float* __restrict__ W, const float* __restrict__ b,
                                                     int E, double* __restrict__ logit, double* __restrict__ absum) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= E) return;
    double acc[MOE_DECODE_MAX_T], ab[MOE_DECODE_MAX_T];
#pragma unroll
    for (int t = 0; t < MOE_DECODE_MAX_T; ++t) acc[t] = ab[t] = 0.0;
    const float4* w4 = reinterpret_cast<const float4*>(W + (size_t)e * H);
#pragma unroll 2
    for (int i = lane; i < H / 4; i += 32) {
        float4 w = __ldg(w4 + i);
        const double w0 = w.x, w1 = w.y, w2 = w.z, w3 = w.w;
#pragma unroll
        for (int t = 0; t < MOE_DECODE_MAX_T; ++t) {
            if (t < T) {
                uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + (size_t)t * H) + i);
                const double x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
                const double x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
                acc[t] = fma(x0, w0, acc[t]);
                acc[t] = fma(x1, w1, acc[t]);
                acc[t] = fma(x2, w2, acc[t]);
                acc[t] = fma(x3, w3, acc[t]);
                ab[t] += fabs(x0 * w0) + fabs(x1 * w1) + fabs(x2 * w2) + fabs(x3 * w3);
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
        double bb = b ? (double)b[e] : 0.0;
        for (int t = 0; t < T; ++t) {
            logit[(size_t)t * E + e] = acc[t] + bb;
            absum[(size_t)t * E + e] = ab[t] + fabs(bb);
        }
    }
}

// ---------------------------------------------------------------- router weight row norms

// wnorm[e] >= ||W[e]||_2 (fp32, inflated by 0.1% to cover its own rounding)
__global__ void k_router_norms(const float* __restrict__ W, int E, int H, float* __restrict__ wnorm) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= E) return;
    const float4* w4 = reinterpret_cast<const float4*>(W + (size_t)e * H);
    float s = 0.f;
    for (int i = lane; i < H / 4; i += 32) {
        float4 w = __ldg(w4 + i);
        s = fmaf(w.x, w.x, fmaf(w.y, w.y, fmaf(w.z, w.z, fmaf(w.w, w.w, s))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) wnorm[e] = sqrtf(s) * 1.001f;
}

// ---------------------------------------------------------------- prefill router: fp32 tiled GEMM

#define RG_BM 128
#define RG_BN 64
#define RG_BK 16

// l[t][e] = sum_h x[t][h] W[e][h] + b_e.  Each output is summed by one thread
// in blocks: 16 products into a fresh partial, partials added in order, then
// the bias, so no product passes through more than 16 + H/16 + 1 roundings.
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
        float part[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
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
                for (int j = 0; j < 4; ++j) part[i][j] = fmaf(a[i], bb[j], part[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
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

// What the fast pass knows about a token it could not certify: its M
// candidates in rank order (value desc, expert asc) and an upper end of
// everything else, so that the slow pass starts at the re-evaluation.
struct SlowRec {
    double val[32];  // fast values
    double bnd[32];  // their error bounds
    int32_t e[32];   // experts
    double rest;     // upper end of every non-candidate (-inf when none)
    int32_t mc;      // number of candidates
    int32_t pad;
};

struct TopkArgs {
    const uint16_t* x;      // [T][H] bf16
    const float* W;         // [E][H]
    const float* b;         // [E] or null
    const void* logit;      // [T][E]: double (decode) or float (prefill) fast logits
    const double* absum;    // decode: [T][E] sums of |x W| + |b|
    const float* xnorm;     // [T] upper bounds of ||x_t||_2, or null (computed here)
    const float* wnorm;     // prefill: [E] upper bounds of ||W[e]||_2
    int32_t* idx;           // [T][k]
    float* w;               // [T][k]
    int32_t* n_rechecked;   // [1]
    int32_t* slow_list;     // tokens the fast pass could not certify (k_topk_fast), or null
    int32_t* slow_count;    // [1] their number (zeroed before the fast pass)
    SlowRec* slow_rec;      // [T] the fast pass's candidates of each listed token
    int32_t* last_list;     // tokens the slow pass could not certify either (k_topk_last)
    int32_t* last_count;    // [1] their number (zeroed before the fast pass)
    double gfast;           // gamma_n of the fast logits' summation
    int T, H, E, k;
};

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ double warp_min_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// The selection order of logits is total: a NaN logit ranks as -inf (below
// every number; ties, as every tie, go to the lower expert index), and an
// error bound that is not a number becomes +inf, against which nothing
// certifies.  Non-finite inputs therefore still give k valid, distinct experts.
__device__ __forceinline__ double order_val(double v) { return isnan(v) ? -INFINITY : v; }
__device__ __forceinline__ double order_bnd(double d) { return isnan(d) ? INFINITY : d; }

// Ends of the interval [v - d, v + d] that holds an exact logit.  An infinite
// bound leaves the value unknown, so its interval is the whole line (plain
// arithmetic would give inf - inf = NaN there, and a NaN end would silently
// drop out of the comparisons, maxima and minima that use it).
__device__ __forceinline__ double lo_end(double v, double d) { return isinf(d) ? -INFINITY : v - d; }
__device__ __forceinline__ double hi_end(double v, double d) { return isinf(d) ? INFINITY : v + d; }

// The definition: fp64, sequential over h, then + b (one thread).
__device__ __forceinline__ double logit_fp64_exact(const TopkArgs& a, int t, int e) {
    const uint16_t* xr = a.x + (size_t)t * a.H;
    const float* wr = a.W + (size_t)e * a.H;
    double s = 0.0;
    // in order over h; 8 elements per step by vector loads (H % 8 == 0, rows 16-byte aligned)
#pragma unroll 4
    for (int h = 0; h < a.H; h += 8) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + h));
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(wr + h));
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(wr + h + 4));
        s = fma((double)__uint_as_float(xv.x << 16), (double)w0.x, s);
        s = fma((double)__uint_as_float(xv.x & 0xffff0000u), (double)w0.y, s);
        s = fma((double)__uint_as_float(xv.y << 16), (double)w0.z, s);
        s = fma((double)__uint_as_float(xv.y & 0xffff0000u), (double)w0.w, s);
        s = fma((double)__uint_as_float(xv.z << 16), (double)w1.x, s);
        s = fma((double)__uint_as_float(xv.z & 0xffff0000u), (double)w1.y, s);
        s = fma((double)__uint_as_float(xv.w << 16), (double)w1.z, s);
        s = fma((double)__uint_as_float(xv.w & 0xffff0000u), (double)w1.w, s);
    }
    if (a.b) s += (double)a.b[e];
    return s;
}

// Lanes j < M hold (cval, cbnd, ce).  Sort them by (cval desc, ce asc); lane r
// receives position r.  Returns whether every decision is certified: each of
// the first k positions is separated from the next, and position k-1 clears
// `rest` (the upper end of everything outside the candidates).
// Exact, order-preserving integer key of a (non-NaN) double: ranking on it is
// ALU work, where chains of fp64 compares cost several times the latency.
__device__ __forceinline__ unsigned long long order_key64(double d) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(d);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// The largest upper end among the candidates ranked k .. M-1 (lanes in rank
// order), rounded up to fp32; -inf when there are none.
__device__ __forceinline__ double tail_hi_end(double cval, double cbnd, int M, int k) {
    const int lane = threadIdx.x & 31;
    const float h = (lane >= k && lane < M) ? __double2float_ru(hi_end(cval, cbnd)) : -INFINITY;
    const uint32_t u = __float_as_uint(h);
    const uint32_t m = __reduce_max_sync(0xffffffffu, (u & 0x80000000u) ? ~u : (u | 0x80000000u));
    return (double)__uint_as_float((m & 0x80000000u) ? (m & 0x7fffffffu) : ~m);
}

// Lanes hold M candidates in (value desc, expert asc) order; `rest` is an upper
// end of every expert that is not a candidate (-inf when there is none).  The
// first k are certified as the exact top k in the exact order when the
// intervals of ranks j and j + 1 are disjoint for j < k - 1 and the lower end
// of rank k - 1 is above the upper end of every candidate ranked k or later
// and above `rest`.
__device__ __forceinline__ bool certify_sorted(double cval, double cbnd, int M, int k, double rest) {
    const int lane = threadIdx.x & 31;
    const double nv = __shfl_down_sync(0xffffffffu, cval, 1);
    const double nb = __shfl_down_sync(0xffffffffu, cbnd, 1);
    const double tail = fmax(rest, tail_hi_end(cval, cbnd, M, k));
    bool ok = true;
    if (lane < k - 1) ok = lo_end(cval, cbnd) > hi_end(nv, nb);
    if (lane == k - 1) ok = lo_end(cval, cbnd) > tail;
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool sort_and_certify(double& cval, double& cbnd, int& ce, int M, int k, double rest) {
    const int lane = threadIdx.x & 31;
    const unsigned long long ck = order_key64(cval);
    const uint32_t ckh = (uint32_t)(ck >> 32), ckl = (uint32_t)ck;
    int rank = 0;
#pragma unroll 8
    for (int j = 0; j < 32; ++j) {
        const uint32_t oh = __shfl_sync(0xffffffffu, ckh, j), ol = __shfl_sync(0xffffffffu, ckl, j);
        const int ej = __shfl_sync(0xffffffffu, ce, j);
        const unsigned long long oj = ((unsigned long long)oh << 32) | ol;
        if (j < M && lane < M && (oj > ck || (oj == ck && ej < ce))) ++rank;
    }
    int src = 0;
    for (int j = 0; j < M; ++j)
        if (__shfl_sync(0xffffffffu, rank, j) == lane) src = j;
    cval = __shfl_sync(0xffffffffu, cval, src);
    cbnd = __shfl_sync(0xffffffffu, cbnd, src);
    ce = __shfl_sync(0xffffffffu, ce, src);
    return certify_sorted(cval, cbnd, M, k, rest);
}

// Lanes hold M candidates in rank order after a failed certification.  The
// candidates to re-evaluate exactly: both ends of every overlapping adjacent
// pair among the k + 1 best, and candidates further down whose interval
// reaches the k-th (which then needs its own value too).  Returns the lane mask.
__device__ __forceinline__ unsigned reeval_mask(double cval, double cbnd, int MC, int k) {
    const int lane = threadIdx.x & 31;
    const double nv = __shfl_down_sync(0xffffffffu, cval, 1);
    const double nb = __shfl_down_sync(0xffffffffu, cbnd, 1);
    const double lok = __shfl_sync(0xffffffffu, lo_end(cval, cbnd), k - 1);
    const bool pairbad = lane < k && lane + 1 < MC && !(lo_end(cval, cbnd) > hi_end(nv, nb));
    const bool tailbad = lane > k && lane < MC && !(lok > hi_end(cval, cbnd));
    const bool anytail = __any_sync(0xffffffffu, tailbad);
    const bool prevup = __shfl_up_sync(0xffffffffu, pairbad ? 1 : 0, 1) != 0;
    const bool prevbad = (prevup && lane > 0) || (lane == k - 1 && anytail);
    return __ballot_sync(0xffffffffu, lane < MC && (pairbad || prevbad || tailbad));
}

// One warp: x_t . W[e] in fp64, lanes taking h = 4 l + 128 i .. + 3 (each lane
// adds H / 32 products), and the sum of the products' magnitudes, both
// reduced over the warp (every lane gets them).
__device__ __forceinline__ void dot_fp64_warp(const TopkArgs& a, int t, int e, double& s, double& sa) {
    const int lane = threadIdx.x & 31, H = a.H;
    const uint16_t* xr = a.x + (size_t)t * H;
    const float* wr = a.W + (size_t)e * H;
    double acc = 0.0, ab = 0.0;
#pragma unroll 4
    for (int h0 = 4 * lane; h0 < H; h0 += 128) {
        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr + h0));
        const float4 wv = __ldg(reinterpret_cast<const float4*>(wr + h0));
        const double p0 = (double)__uint_as_float(xv.x << 16) * (double)wv.x;
        const double p1 = (double)__uint_as_float(xv.x & 0xffff0000u) * (double)wv.y;
        const double p2 = (double)__uint_as_float(xv.y << 16) * (double)wv.z;
        const double p3 = (double)__uint_as_float(xv.y & 0xffff0000u) * (double)wv.w;
        acc += p0; acc += p1; acc += p2; acc += p3;
        ab += fabs(p0); ab += fabs(p1); ab += fabs(p2); ab += fabs(p3);
    }
    s = warp_sum_d(acc);
    sa = warp_sum_d(ab);
}

__device__ __forceinline__ void write_topk(int k, double cval, int ce, int32_t* idx_out, float* w_out) {
    const int lane = threadIdx.x & 31;
    const double v0 = __shfl_sync(0xffffffffu, cval, 0);
    const float z = (lane < k) ? expf((float)(cval - v0)) : 0.f;  // differences are small: fp32 exp suffices
    float zs = z;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
    if (lane < k) {
        idx_out[lane] = ce;
        w_out[lane] = z / zs;
    }
}

// Top-k of token t by one warp; lanes hold the fast logits of experts
// e = lane + 32 i.  Results go to idx_out[0..k) / w_out[0..k); cs / cvs are
// per-warp scratch of MOE_MAX_E entries for the exact path.
// MODE 0: fp32 logits, bound from norms (prefill); 1: fp64 logits with
// per-entry sums of |x W| (decode kernels); 2: fp64 logits, bound from norms
// (fused decode, whose router runs on the fp64 tensor cores).
// FAST_ONLY: a token whose fast values do not certify is appended to
// a.slow_list (for k_topk_slow) instead of being finished here, which keeps the
// fp64 re-evaluation's registers out of the common pass.
template <int MODE, bool FAST_ONLY = false>
__device__ __forceinline__ void topk_token(const TopkArgs& a, int t, int32_t* idx_out, float* w_out, int* cs,
                                           double* cvs, int32_t* nrechk) {
    constexpr bool F64 = MODE != 0;
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k, H = a.H;
    constexpr int NV = MOE_MAX_E / 32;
    const double u64 = 1.1102230246251565e-16;            // 2^-53
    const double g_or = (double)(H + 2) * u64 * 1.01;     // the definition's own rounding, per unit of B
    const double g_par = (double)(H / 32 + 8) * u64 * 1.01;  // warp-parallel fp64 sums

    float xnorm = 0.f;
    if (MODE != 1) {  // ||x_t||_2, inflated to cover its fp32 rounding
        if (a.xnorm) {
            xnorm = a.xnorm[t];
        } else {
            const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * H);
            float s = 0.f;
            for (int i = lane; i < H / 8; i += 32) {
                const uint4 r = __ldg(xr + i);
                const uint32_t wd[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    const float lo = __uint_as_float(wd[z] << 16), hi = __uint_as_float(wd[z] & 0xffff0000u);
                    s = fmaf(lo, lo, fmaf(hi, hi, s));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            xnorm = sqrtf(s) * 1.001f;
        }
    }
    // fp32 fast logits (MODE 0) are held in fp32 with their bounds rounded up to
    // fp32: half the registers of fp64 values, and the intervals only widen
    using VT = typename std::conditional<F64, double, float>::type;
    VT v[NV], dl[NV];
    uint32_t key[NV];  // order-preserving 32-bit keys of the values rounded to fp32
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            double B;
            float f;
            if (F64) {
                v[i] = order_val(static_cast<const double*>(a.logit)[(size_t)t * E + e]);
                f = (float)v[i];
            } else {
                f = static_cast<const float*>(a.logit)[(size_t)t * E + e];
                if (isnan(f)) f = -INFINITY;
                v[i] = f;
            }
            if (MODE == 1) B = a.absum[(size_t)t * E + e] * (1.0 + 1e-9);
            else B = ((double)xnorm * (double)a.wnorm[e] + (a.b ? fabs((double)a.b[e]) : 0.0)) * 1.001;
            const double bd = order_bnd(B * (a.gfast + g_or) + 1e-300);
            dl[i] = F64 ? (VT)bd : (VT)__double2float_ru(bd);
            const uint32_t u = __float_as_uint(f);
            key[i] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        } else {
            v[i] = -INFINITY;
            dl[i] = 0.0;
            key[i] = 0;
            taken |= 1u << i;
        }
    }
    // 1) Candidates by the 32-bit keys; a candidate set that misses a member of
    //    the true top k only fails the certification below.  First try every
    //    entry at or above theta, the M-th largest of the 32 lane maxima: at
    //    least M entries (those maxima) reach theta, so this set holds the M
    //    largest.  With more than 32 of them, pick exactly M by M rounds of
    //    warp-wide argmax.
    const int M = min(min(E, k + MOE_CAND_EXTRA), 32);
    int ce = -1;
    double cval = -INFINITY, cbnd = 0.0;
    int MC = M;  // candidates held one per lane
    bool picked = false;  // warp-uniform: the threshold set was taken
    {
        uint32_t lmax = 0;  // invalid entries are marked taken and have key 0
#pragma unroll
        for (int i = 0; i < NV; ++i)
            if (!((taken >> i) & 1u)) lmax = max(lmax, key[i]);
        int r = 0;
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
            const uint32_t o = __shfl_sync(0xffffffffu, lmax, j);
            r += (o > lmax || (o == lmax && j < lane)) ? 1 : 0;
        }
        const uint32_t thk = __shfl_sync(0xffffffffu, lmax, __ffs(__ballot_sync(0xffffffffu, r == M - 1)) - 1);
        unsigned bm[NV];
        int nc = 0;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            bm[i] = __ballot_sync(0xffffffffu, !((taken >> i) & 1u) && key[i] >= thk);
            nc += __popc(bm[i]);
        }
        if (nc <= 32) {
            int base = 0;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                if ((bm[i] >> lane) & 1u) {
                    const int pos = base + __popc(bm[i] & ((1u << lane) - 1));
                    cs[pos] = lane + 32 * i;
                    cvs[pos] = v[i];
                    cvs[32 + pos] = dl[i];
                }
                base += __popc(bm[i]);
            }
            __syncwarp();
            if (lane < nc) {
                ce = cs[lane];
                cval = cvs[lane];
                cbnd = cvs[32 + lane];
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < NV; ++i) taken |= ((bm[i] >> lane) & 1u) << i;
            MC = nc;
            picked = true;
        }
    }
    if (!picked) {  // the threshold set was too large: M rounds of argmax
        uint32_t lkey = 0;
        int li = -1;
        auto rescan = [&]() {  // this lane's best untaken entry (lowest index on equal keys)
            lkey = 0;
            li = -1;
#pragma unroll
            for (int i = 0; i < NV; ++i)
                if (!((taken >> i) & 1u) && (li < 0 || key[i] > lkey)) { lkey = key[i]; li = i; }
        };
        rescan();
        for (int j = 0; j < M; ++j) {
            const uint32_t mk = __reduce_max_sync(0xffffffffu, lkey);
            const uint32_t me =
                __reduce_min_sync(0xffffffffu, (li >= 0 && lkey == mk) ? (uint32_t)(lane + 32 * li) : 0xffffffffu);
            const int owner = (int)(me & 31u);
            double lv = 0.0, ld = 0.0;
            if (lane == owner) {
#pragma unroll
                for (int i = 0; i < NV; ++i)
                    if (i == li) { lv = v[i]; ld = dl[i]; }
            }
            const double bv = __shfl_sync(0xffffffffu, lv, owner);
            const double bd = __shfl_sync(0xffffffffu, ld, owner);
            if (lane == j) { ce = (int)me; cval = bv; cbnd = bd; }
            if (lane == owner) {
                taken |= 1u << li;
                rescan();
            }
        }
    }
    float rest_f = -INFINITY;  // an upper end of everything left out, rounded up to fp32 (a short fp32 chain)
#pragma unroll
    for (int i = 0; i < NV; ++i)
        if (!((taken >> i) & 1u)) rest_f = fmaxf(rest_f, __double2float_ru(hi_end(v[i], dl[i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rest_f = fmaxf(rest_f, __shfl_xor_sync(0xffffffffu, rest_f, o));
    const double rest = (double)rest_f;

    // 2) certified on the fast values?
    if (sort_and_certify(cval, cbnd, ce, MC, k, rest)) {
        write_topk(k, cval, ce, idx_out, w_out);
        return;
    }
    if (FAST_ONLY) {
        int slot = 0;
        if (lane == 0) {
            slot = atomicAdd(a.slow_count, 1);
            a.slow_list[slot] = t;
        }
        slot = __shfl_sync(0xffffffffu, slot, 0);
        SlowRec* r = a.slow_rec + slot;
        r->val[lane] = cval;
        r->bnd[lane] = cbnd;
        r->e[lane] = ce;
        if (lane == 0) {
            r->rest = rest;
            r->mc = MC;
        }
        return;
    }
    // 3) prefill: re-evaluate in fp64 (lane-strided) the candidates that the
    //    certification could not separate: both ends of every overlapping
    //    adjacent pair among the k + 1 best (the lanes are in rank order after
    //    sort_and_certify).  The others keep their fast values and bounds,
    //    which still contain the exact logits, so the second certification
    //    below is as valid as the first.
    if (MODE == 0) {
        const unsigned need = reeval_mask(cval, cbnd, MC, k);
        const int NR = __popc(need);
        for (int base = 0; base < NR; base += 16) {
            int ej[16], lj[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {  // lane of the (base + j)-th flagged candidate
                unsigned mm = need;
                for (int z = 0; z < base + j && mm; ++z) mm &= mm - 1;
                lj[j] = mm ? __ffs(mm) - 1 : 31;
                ej[j] = __shfl_sync(0xffffffffu, ce, lj[j]);
            }
            double acc[16], ab[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = ab[j] = 0.0;
            const uint16_t* xr = a.x + (size_t)t * H;
            // lane l takes h = 4 l + 128 i .. + 3 (H % 4 == 0, rows 16-byte aligned): one
            // 8-byte x load and one 16-byte row load per candidate keep all of a step's
            // loads in flight; each lane still adds H / 32 products
            for (int h0 = 4 * lane; h0 < H; h0 += 128) {
                const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr + h0));
                const double x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
                const double x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
                float4 wv[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (base + j < NR) wv[j] = __ldg(reinterpret_cast<const float4*>(a.W + (size_t)ej[j] * H + h0));
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (base + j < NR) {
                        const double p0 = x0 * (double)wv[j].x, p1 = x1 * (double)wv[j].y;
                        const double p2 = x2 * (double)wv[j].z, p3 = x3 * (double)wv[j].w;
                        acc[j] += p0; acc[j] += p1; acc[j] += p2; acc[j] += p3;
                        ab[j] += fabs(p0); ab[j] += fabs(p1); ab[j] += fabs(p2); ab[j] += fabs(p3);
                    }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (base + j < NR) {
                    const double s = warp_sum_d(acc[j]), sa = warp_sum_d(ab[j]);
                    const double bb = a.b ? (double)a.b[ej[j]] : 0.0;
                    if (lane == lj[j]) {
                        cval = order_val(s + bb);
                        cbnd = order_bnd((sa + fabs(bb)) * (1.0 + 1e-9) * (g_par + g_or) + 1e-300);
                    }
                }
            }
        }
        if (sort_and_certify(cval, cbnd, ce, MC, k, rest)) {
            write_topk(k, cval, ce, idx_out, w_out);
            return;
        }
    }
    // 4) exact: every expert whose upper end reaches theta (the lowest lower
    //    end among the k best) is evaluated by the definition itself
    const double th = warp_min_d(lane < k ? lo_end(cval, cbnd) : INFINITY);
    int nc = 0;
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        // the step-1 candidates (marked taken) are always kept
        const bool in = (e < E) && ((((taken >> i) & 1u) != 0) || hi_end(v[i], dl[i]) >= th);
        const unsigned m = __ballot_sync(0xffffffffu, in);
        if (in) cs[nc + __popc(m & ((1u << lane) - 1))] = e;
        nc += __popc(m);
    }
    __syncwarp();
    for (int c = lane; c < nc; c += 32) cvs[c] = order_val(logit_fp64_exact(a, t, cs[c]));
    __syncwarp();
    double l0 = 0.0, z = 0.0, mine = 0.0;
    for (int j = 0; j < k; ++j) {
        double bv = -INFINITY;
        int be = 0x7fffffff, bc = -1;
        for (int c = lane; c < nc; c += 32)
            if (cs[c] >= 0 && (cvs[c] > bv || (cvs[c] == bv && cs[c] < be))) { bv = cvs[c]; be = cs[c]; bc = c; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            double v2 = __shfl_xor_sync(0xffffffffu, bv, o);
            int e2 = __shfl_xor_sync(0xffffffffu, be, o);
            int c2 = __shfl_xor_sync(0xffffffffu, bc, o);
            if (v2 > bv || (v2 == bv && e2 < be)) { bv = v2; be = e2; bc = c2; }
        }
        __syncwarp();
        if (lane == 0) {
            // at least k candidates and a total order: bc is always found; the
            // guard only keeps a library fault from writing outside the arrays
            if (bc >= 0 && be < E) {
                cs[bc] = -1;  // taken
                idx_out[j] = be;
            } else {
                idx_out[j] = 0;
                moe_set_status(MOE_ERR_RANGE);
            }
        }
        __syncwarp();
        if (j == 0) l0 = bv;
        const double zz = (double)expf((float)(bv - l0));
        z += zz;
        if (lane == j) mine = zz;
    }
    if (lane < k) w_out[lane] = (float)(mine / z);
    if (lane == 0 && nrechk) atomicAdd(nrechk, 1);
}

// ||x_t||_2 of every token, inflated to cover its fp32 rounding; one warp per token.
__global__ void __launch_bounds__(256) k_xnorm(const uint16_t* __restrict__ x, int T, int H, float* __restrict__ xn) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    float s = 0.f;
#pragma unroll 8
    for (int i = lane; i < H / 8; i += 32) {
        const uint4 r = __ldg(xr + i);
        const uint32_t wd[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
            const float lo = __uint_as_float(wd[z] << 16), hi = __uint_as_float(wd[z] & 0xffff0000u);
            s = fmaf(lo, lo, fmaf(hi, hi, s));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) xn[t] = sqrtf(s) * 1.001f;
}

// One warp per token: the fast pass; tokens it cannot certify go to k_topk_slow.
template <int MODE>
__global__ void __launch_bounds__(32 * MOE_TOPK_WARPS) k_topk_fast(TopkArgs a) {
    __shared__ int s_ce[MOE_TOPK_WARPS][64];
    __shared__ double s_cv[MOE_TOPK_WARPS][64];
    const int wid = threadIdx.x >> 5;
    const int t = blockIdx.x * MOE_TOPK_WARPS + wid;
    if (t >= a.T) return;
    topk_token<MODE, true>(a, t, a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k, s_ce[wid], s_cv[wid], a.n_rechecked);
}

// The tokens k_topk_fast listed (prefill fast logits), one CTA each, looping
// over the list: warp 0 takes the fast pass's ranked candidates and flags the
// ones to re-evaluate, every warp re-evaluates some of them in fp64, and warp 0
// certifies again; a token that still does not certify goes to k_topk_last.
#define MOE_SLOW_WARPS 8
__global__ void __launch_bounds__(32 * MOE_SLOW_WARPS) k_topk_slow(TopkArgs a) {
    __shared__ int s_list[32];
    __shared__ int s_e[32];
    __shared__ double s_v[32], s_b[32];
    __shared__ int s_nr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const double u64 = 1.1102230246251565e-16;
    const double g_or = (double)(a.H + 2) * u64 * 1.01;         // the definition's own rounding
    const double g_par = (double)(a.H / 32 + 8) * u64 * 1.01;   // warp-parallel fp64 sums
    const int n = *a.slow_count;
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const int t = a.slow_list[i];
        const SlowRec* r = a.slow_rec + i;
        double cval = -INFINITY, cbnd = 0.0;
        int ce = 0x7fffffff, MC = 0;
        double rest = 0.0;
        if (warp == 0) {
            MC = r->mc;
            rest = r->rest;
            if (lane < MC) {
                cval = r->val[lane];
                cbnd = r->bnd[lane];
                ce = r->e[lane];
            }
            const unsigned need = reeval_mask(cval, cbnd, MC, a.k);
            if ((need >> lane) & 1u) s_list[__popc(need & ((1u << lane) - 1))] = lane;
            s_e[lane] = ce;
            if (lane == 0) s_nr = __popc(need);
        }
        __syncthreads();
        const int NR = s_nr;
        for (int q = warp; q < NR; q += MOE_SLOW_WARPS) {
            const int j = s_list[q], e = s_e[j];
            double sm, sa;
            dot_fp64_warp(a, t, e, sm, sa);
            if (lane == 0) {
                const double bb = a.b ? (double)a.b[e] : 0.0;
                s_v[j] = order_val(sm + bb);
                s_b[j] = order_bnd((sa + fabs(bb)) * (1.0 + 1e-9) * (g_par + g_or) + 1e-300);
            }
        }
        __syncthreads();
        if (warp == 0) {
            for (int q = 0; q < NR; ++q)
                if (s_list[q] == lane) {
                    cval = s_v[lane];
                    cbnd = s_b[lane];
                }
            if (sort_and_certify(cval, cbnd, ce, MC, a.k, rest))
                write_topk(a.k, cval, ce, a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k);
            else if (lane == 0)
                a.last_list[atomicAdd(a.last_count, 1)] = t;
        }
        __syncthreads();  // the shared lists are reused by the next token
    }
}

// The tokens k_topk_slow could not certify, one warp each: the whole
// single-warp path of topk_token, its exact fallback included.
__global__ void __launch_bounds__(32 * MOE_TOPK_WARPS) k_topk_last(TopkArgs a) {
    __shared__ int s_ce[MOE_TOPK_WARPS][MOE_MAX_E];
    __shared__ double s_cv[MOE_TOPK_WARPS][MOE_MAX_E];
    const int wid = threadIdx.x >> 5;
    const int i = blockIdx.x * MOE_TOPK_WARPS + wid;
    if (i >= *a.last_count) return;
    const int t = a.last_list[i];
    topk_token<0>(a, t, a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k, s_ce[wid], s_cv[wid], a.n_rechecked);
}

// One warp per token.
template <int MODE>
__global__ void __launch_bounds__(32 * MOE_TOPK_WARPS) k_topk(TopkArgs a) {
    __shared__ int s_ce[MOE_TOPK_WARPS][MOE_MAX_E];
    __shared__ double s_cv[MOE_TOPK_WARPS][MOE_MAX_E];
    const int wid = threadIdx.x >> 5;
    const int t = blockIdx.x * MOE_TOPK_WARPS + wid;
    if (t >= a.T) return;
    topk_token<MODE>(a, t, a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k, s_ce[wid], s_cv[wid], a.n_rechecked);
}
