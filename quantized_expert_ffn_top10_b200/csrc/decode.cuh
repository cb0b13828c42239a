// Decode path (T <= MOE_DECODE_MAX_T): the experts selected by the window are
// streamed once each.  For every selected expert e with tokens t_1..t_n:
//   gate/up: g_j[r] = W_g[r] . x_{t_j}, u_j[r] = W_u[r] . x_{t_j},
//            h_j[r] = silu(g_j[r]) * u_j[r]              (fp32, exact dequant)
//   down:    y_j[c] = w_j * (W_d[c] . h_j)                (fp32)
// then out[t] = (residual ? x_t : 0) + sum_j y_{pair(t, j)} in slot order.
// Each warp owns whole rows; a lane takes 8 consecutive elements of every
// 256-element chunk, so one warp load moves 128 contiguous bytes of 4-bit
// codes (64 of 2-bit) and the scale of a 32-element block is applied to the
// partial sums of the four lanes that share it.
#pragma once
#include "common.cuh"

struct DecodeArgs {
    const uint8_t* arena;
    const int32_t* slot_table;  // [L][E]
    int64_t slot_bytes, n_slots;
    int64_t off_codes[3], off_scales[3];
    int H, I, E, k, layer;
    const uint16_t* x;     // [T][H]
    const int32_t* offsets;
    const int32_t* perm;
    const int32_t* uniq;
    const int32_t* meta;   // [0] = number of selected experts
    const float* topk_w;   // [T*k]
    float* h;              // [P][I] workspace
    float* y;              // [P][H] workspace
};

// 8 codes of b bits starting at element c0 (c0 % 8 == 0) of a packed row.
template <int BITS>
__device__ __forceinline__ uint32_t load8(const uint8_t* row, int c0) {
    if (BITS == 4) return __ldg(reinterpret_cast<const uint32_t*>(row + c0 / 2));
    return __ldg(reinterpret_cast<const uint16_t*>(row + c0 / 4));
}

template <int BITS>
__device__ __forceinline__ float code_at(uint32_t w, int i) {
    return (float)((int)((w >> (i * BITS)) & ((1u << BITS) - 1)) - (1 << (BITS - 1)));
}

// partial dot of 8 codes (offset removed) with 8 values
template <int BITS>
__device__ __forceinline__ float dot8(uint32_t w, const float (&v)[8]) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s = fmaf(code_at<BITS>(w, i), v[i], s);
    return s;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 q, float (&v)[8]) {
    v[0] = __uint_as_float(q.x << 16); v[1] = __uint_as_float(q.x & 0xffff0000u);
    v[2] = __uint_as_float(q.y << 16); v[3] = __uint_as_float(q.y & 0xffff0000u);
    v[4] = __uint_as_float(q.z << 16); v[5] = __uint_as_float(q.z & 0xffff0000u);
    v[6] = __uint_as_float(q.w << 16); v[7] = __uint_as_float(q.w & 0xffff0000u);
}

// remote: the slot-table entry is MOE_SLOT_REMOTE (held by another GPU, not an error)
__device__ __forceinline__ const uint8_t* expert_slot(const DecodeArgs& a, int e, bool& ok, bool& remote) {
    int64_t s = a.slot_table[(int64_t)a.layer * a.E + e];
    ok = (s >= 0 && s < a.n_slots);
    remote = s == MOE_SLOT_REMOTE;
    return ok ? a.arena + s * a.slot_bytes : nullptr;
}

#define DEC_GU_WARPS 16
#define DEC_GU_ROWS_PER_WARP 2

// grid (ceil(I / 32), E_max), block 512; dynamic smem: n_e * H bf16
template <int BG, int BU>
__global__ void __launch_bounds__(32 * DEC_GU_WARPS) k_dec_gateup(DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t dsm[];
    uint16_t* xs = reinterpret_cast<uint16_t*>(dsm);
    if ((int)blockIdx.y >= a.meta[0]) return;
    const int e = a.uniq[blockIdx.y];
    const int r0 = a.offsets[e], n = a.offsets[e + 1] - r0;
    const int H = a.H, I = a.I;
    bool ok, remote;
    const uint8_t* slot = expert_slot(a, e, ok, remote);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (!ok) {  // no valid slot: this expert contributes zero
        if (threadIdx.x == 0 && blockIdx.x == 0 && !remote) moe_set_status(MOE_ERR_SLOT);
        for (int r = blockIdx.x * 32 + threadIdx.x; r < min(I, (int)(blockIdx.x + 1) * 32); r += blockDim.x)
            for (int j = 0; j < n; ++j) a.h[(size_t)(r0 + j) * I + r] = 0.f;
        return;
    }
    for (int i = threadIdx.x; i < n * H / 8; i += blockDim.x) {
        int j = i / (H / 8), c = i % (H / 8);
        int t = a.perm[r0 + j] / a.k;
        reinterpret_cast<uint4*>(xs)[i] = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * H) + c);
    }
    __syncthreads();
    const uint8_t* cg = slot + a.off_codes[0];
    const uint8_t* cu = slot + a.off_codes[1];
    const uint16_t* sg = reinterpret_cast<const uint16_t*>(slot + a.off_scales[0]);
    const uint16_t* su = reinterpret_cast<const uint16_t*>(slot + a.off_scales[1]);
    for (int rr = 0; rr < DEC_GU_ROWS_PER_WARP; ++rr) {
        const int r = blockIdx.x * 32 + wid * DEC_GU_ROWS_PER_WARP + rr;
        if (r >= I) break;
        const uint8_t* rowg = cg + (size_t)r * H * BG / 8;
        const uint8_t* rowu = cu + (size_t)r * H * BU / 8;
        float g[MOE_DECODE_MAX_T], u[MOE_DECODE_MAX_T];
#pragma unroll
        for (int j = 0; j < MOE_DECODE_MAX_T; ++j) g[j] = u[j] = 0.f;
        for (int c0 = lane * 8; c0 < H; c0 += 256) {
            uint32_t wg = load8<BG>(rowg, c0), wu = load8<BU>(rowu, c0);
            float s_g = half_bits_to_f32(__ldg(sg + (size_t)r * (H / 32) + c0 / 32));
            float s_u = half_bits_to_f32(__ldg(su + (size_t)r * (H / 32) + c0 / 32));
#pragma unroll
            for (int j = 0; j < MOE_DECODE_MAX_T; ++j) {
                if (j < n) {
                    float xv[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4*>(xs + (size_t)j * H + c0), xv);
                    g[j] = fmaf(s_g, dot8<BG>(wg, xv), g[j]);
                    u[j] = fmaf(s_u, dot8<BU>(wu, xv), u[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < MOE_DECODE_MAX_T; ++j) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                g[j] += __shfl_xor_sync(0xffffffffu, g[j], o);
                u[j] += __shfl_xor_sync(0xffffffffu, u[j], o);
            }
        }
        if (lane == 0)
            for (int j = 0; j < n; ++j) a.h[(size_t)(r0 + j) * I + r] = silu_f32(g[j]) * u[j];
    }
}

#define DEC_DN_WARPS 16
#define DEC_DN_ROWS_PER_WARP 2

// grid (ceil(H / 32), E_max), block 512; dynamic smem: n_e * I fp32
template <int BD>
__global__ void __launch_bounds__(32 * DEC_DN_WARPS) k_dec_down(DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t dsm[];
    float* hs = reinterpret_cast<float*>(dsm);
    if ((int)blockIdx.y >= a.meta[0]) return;
    const int e = a.uniq[blockIdx.y];
    const int r0 = a.offsets[e], n = a.offsets[e + 1] - r0;
    const int H = a.H, I = a.I;
    bool ok, remote;
    const uint8_t* slot = expert_slot(a, e, ok, remote);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (!ok) {
        for (int c = blockIdx.x * 32 + threadIdx.x; c < min(H, (int)(blockIdx.x + 1) * 32); c += blockDim.x)
            for (int j = 0; j < n; ++j) a.y[(size_t)(r0 + j) * H + c] = 0.f;
        return;
    }
    for (int i = threadIdx.x; i < n * I; i += blockDim.x) hs[i] = a.h[(size_t)r0 * I + i];
    __syncthreads();
    const uint8_t* cd = slot + a.off_codes[2];
    const uint16_t* sd = reinterpret_cast<const uint16_t*>(slot + a.off_scales[2]);
    float wj[MOE_DECODE_MAX_T];
#pragma unroll
    for (int j = 0; j < MOE_DECODE_MAX_T; ++j) wj[j] = (j < n) ? a.topk_w[a.perm[r0 + j]] : 0.f;
    for (int rr = 0; rr < DEC_DN_ROWS_PER_WARP; ++rr) {
        const int c = blockIdx.x * 32 + wid * DEC_DN_ROWS_PER_WARP + rr;
        if (c >= H) break;
        const uint8_t* row = cd + (size_t)c * I * BD / 8;
        float acc[MOE_DECODE_MAX_T];
#pragma unroll
        for (int j = 0; j < MOE_DECODE_MAX_T; ++j) acc[j] = 0.f;
        for (int c0 = lane * 8; c0 < I; c0 += 256) {
            uint32_t wd = load8<BD>(row, c0);
            float s = half_bits_to_f32(__ldg(sd + (size_t)c * (I / 32) + c0 / 32));
#pragma unroll
            for (int j = 0; j < MOE_DECODE_MAX_T; ++j) {
                if (j < n) {
                    float hv[8];
                    const float4* hp = reinterpret_cast<const float4*>(hs + (size_t)j * I + c0);
                    float4 h0 = hp[0], h1 = hp[1];
                    hv[0] = h0.x; hv[1] = h0.y; hv[2] = h0.z; hv[3] = h0.w;
                    hv[4] = h1.x; hv[5] = h1.y; hv[6] = h1.z; hv[7] = h1.w;
                    acc[j] = fmaf(s, dot8<BD>(wd, hv), acc[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < MOE_DECODE_MAX_T; ++j)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
        if (lane == 0)
            for (int j = 0; j < n; ++j) a.y[(size_t)(r0 + j) * H + c] = wj[j] * acc[j];
    }
}

// out[t][c] = bf16((residual ? x[t][c] : 0) + sum_j y[inv[t*k + j]][c]), fp32, j in order.
// Y is fp32 (decode) or bf16 (prefill).
template <typename YT>
__global__ void k_combine(const uint16_t* __restrict__ x, const YT* __restrict__ y, const int32_t* __restrict__ inv,
                          int T, int H, int k, int residual, uint16_t* __restrict__ out) {
    const int t = blockIdx.y;
    const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (t >= T || c >= H) return;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
        const size_t row = (size_t)inv[(size_t)t * k + j] * H + c;
        if constexpr (sizeof(YT) == 4) {
            float4 v = __ldg(reinterpret_cast<const float4*>(y + row));
            acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
        } else {
            uint2 v = __ldg(reinterpret_cast<const uint2*>(y + row));
            acc[0] += __uint_as_float(v.x << 16); acc[1] += __uint_as_float(v.x & 0xffff0000u);
            acc[2] += __uint_as_float(v.y << 16); acc[3] += __uint_as_float(v.y & 0xffff0000u);
        }
    }
    if (residual) {
        uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + (size_t)t * H + c));
        acc[0] += __uint_as_float(xv.x << 16); acc[1] += __uint_as_float(xv.x & 0xffff0000u);
        acc[2] += __uint_as_float(xv.y << 16); acc[3] += __uint_as_float(xv.y & 0xffff0000u);
    }
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_bits(acc[0]) | ((uint32_t)f32_to_bf16_bits(acc[1]) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(acc[2]) | ((uint32_t)f32_to_bf16_bits(acc[3]) << 16);
    *reinterpret_cast<uint2*>(out + (size_t)t * H + c) = o;
}


// Partial combine (expert parallelism): part[t][c] = sum_j y[inv[t*k + j]][c]
// in fp32, j in order, no residual and no rounding.  y is fp32 (decode) or
// bf16 (prefill); rows of remote experts are zero.
template <typename YT>
__global__ void k_combine_f32(const YT* __restrict__ y, const int32_t* __restrict__ inv, int T, int H, int k,
                              float* __restrict__ part) {
    const int t = blockIdx.y;
    const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (t >= T || c >= H) return;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
        const size_t row = (size_t)inv[(size_t)t * k + j] * H + c;
        if constexpr (sizeof(YT) == 4) {
            float4 v = __ldg(reinterpret_cast<const float4*>(y + row));
            acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
        } else {
            uint2 v = __ldg(reinterpret_cast<const uint2*>(y + row));
            acc[0] += __uint_as_float(v.x << 16); acc[1] += __uint_as_float(v.x & 0xffff0000u);
            acc[2] += __uint_as_float(v.y << 16); acc[3] += __uint_as_float(v.y & 0xffff0000u);
        }
    }
    *reinterpret_cast<float4*>(part + (size_t)t * H + c) = make_float4(acc[0], acc[1], acc[2], acc[3]);
}

// Prefill combine for bf16 Y: out[t][c..c+7] = sum_j Y[inv[t][j]][c..c+7] (+ x),
// summed in j order in fp32; 16-byte loads, four rows in flight.
__global__ void __launch_bounds__(128) k_combine_bf16x8(const uint16_t* __restrict__ x, const uint16_t* __restrict__ y,
                                                        const int32_t* __restrict__ inv, int T, int H, int k,
                                                        int residual, uint16_t* __restrict__ out) {
    const int t = blockIdx.y;
    const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (t >= T || c >= H) return;
    float acc[8];
#pragma unroll
    for (int z = 0; z < 8; ++z) acc[z] = 0.f;
    const int32_t* iv = inv + (size_t)t * k;
    for (int j0 = 0; j0 < k; j0 += 4) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j0 + j < k) v[j] = __ldg(reinterpret_cast<const uint4*>(y + (size_t)__ldg(iv + j0 + j) * H + c));
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j0 + j < k) {
                const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    acc[2 * z] += __uint_as_float(w[z] << 16);
                    acc[2 * z + 1] += __uint_as_float(w[z] & 0xffff0000u);
                }
            }
    }
    if (residual) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + c));
        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
            acc[2 * z] += __uint_as_float(w[z] << 16);
            acc[2 * z + 1] += __uint_as_float(w[z] & 0xffff0000u);
        }
    }
    uint4 o;
    o.x = (uint32_t)f32_to_bf16_bits(acc[0]) | ((uint32_t)f32_to_bf16_bits(acc[1]) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(acc[2]) | ((uint32_t)f32_to_bf16_bits(acc[3]) << 16);
    o.z = (uint32_t)f32_to_bf16_bits(acc[4]) | ((uint32_t)f32_to_bf16_bits(acc[5]) << 16);
    o.w = (uint32_t)f32_to_bf16_bits(acc[6]) | ((uint32_t)f32_to_bf16_bits(acc[7]) << 16);
    *reinterpret_cast<uint4*>(out + (size_t)t * H + c) = o;
}

// ---------------------------------------------------------------- steering projection

// The steering projection of the "Coder benchmark record" page (steering
// vector section): the layer's output row h (residual included, fp32) loses
// its component along the unit direction v, out = bf16(h - (h . v) v), with v
// used as given.  One block per token.  h is either summed here from the
// per-pair outputs y (fp32 or bf16, in slot order, then + x, as the plain
// combine does) or read from hsrc; the dot product is summed in a fixed order
// (each thread over its features in order, a fixed shuffle tree, the warps in
// order), so repeated calls are bit-identical.
#define STEER_THREADS 256

template <typename YT>
__global__ void __launch_bounds__(STEER_THREADS)
    k_combine_steer(const uint16_t* __restrict__ x, const YT* __restrict__ y, const int32_t* __restrict__ inv,
                    const float* __restrict__ hsrc, int T, int H, int k, int residual, const float* __restrict__ v,
                    uint16_t* __restrict__ out) {
    extern __shared__ float s_h[];  // [H]
    __shared__ float s_red[STEER_THREADS / 32 + 1];
    const int t = blockIdx.x;
    if (t >= T) return;
    float part = 0.f;
    for (int c = threadIdx.x; c < H; c += STEER_THREADS) {
        float h;
        if (hsrc) {
            h = hsrc[(size_t)t * H + c];
        } else {
            float acc = 0.f;
            for (int j = 0; j < k; ++j) {
                const size_t i = (size_t)inv[(size_t)t * k + j] * H + c;
                if constexpr (sizeof(YT) == 4) acc += (float)y[i];
                else acc += bf16_bits_to_f32((uint16_t)y[i]);
            }
            h = residual ? acc + bf16_bits_to_f32(x[(size_t)t * H + c]) : acc;
        }
        s_h[c] = h;
        part = fmaf(h, v[c], part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
        float d = 0.f;
        for (int w = 0; w < STEER_THREADS / 32; ++w) d += s_red[w];
        s_red[STEER_THREADS / 32] = d;
    }
    __syncthreads();
    const float dot = s_red[STEER_THREADS / 32];
    for (int c = threadIdx.x; c < H; c += STEER_THREADS)
        out[(size_t)t * H + c] = f32_to_bf16_bits(fmaf(-dot, v[c], s_h[c]));
}

// The finishing step of an expert-parallel layer: out[t] = bf16(r) with
// r = (residual ? x[t] : 0) + sum[t] in fp32, projected first when v != NULL
// (r - (r . v) v, the dot product summed in a fixed order as in
// k_combine_steer).  One block per token.
__global__ void __launch_bounds__(STEER_THREADS)
    k_finish_rows(const uint16_t* __restrict__ x, const float* __restrict__ sum, int T, int H, int residual,
                  const float* __restrict__ v, uint16_t* __restrict__ out) {
    extern __shared__ float s_r[];  // [H]
    __shared__ float s_red[STEER_THREADS / 32 + 1];
    const int t = blockIdx.x;
    if (t >= T) return;
    float part = 0.f;
    for (int c = threadIdx.x; c < H; c += STEER_THREADS) {
        const float sv = sum[(size_t)t * H + c];
        const float r = residual ? sv + bf16_bits_to_f32(x[(size_t)t * H + c]) : sv;
        s_r[c] = r;
        if (v) part = fmaf(r, v[c], part);
    }
    float dot = 0.f;
    if (v) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = part;
        __syncthreads();
        if (threadIdx.x == 0) {
            float d = 0.f;
            for (int w = 0; w < STEER_THREADS / 32; ++w) d += s_red[w];
            s_red[STEER_THREADS / 32] = d;
        }
        __syncthreads();
        dot = s_red[STEER_THREADS / 32];
    }
    for (int c = threadIdx.x; c < H; c += STEER_THREADS)
        out[(size_t)t * H + c] = f32_to_bf16_bits(v ? fmaf(-dot, v[c], s_r[c]) : s_r[c]);
}
