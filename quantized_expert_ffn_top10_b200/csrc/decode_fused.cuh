// Decode window (T <= 8 tokens) as one persistent, cooperatively launched
// kernel per layer: one CTA per SM, two grid-wide barriers.
//
//   A  router logits in fp64 (warp per expert, experts spread over all SMs)
//   -- barrier --
//   B  every CTA certifies the top-k of every token (the same deterministic
//      computation everywhere, so no second barrier is needed) and builds
//      the grouping (pairs sorted by expert) in shared memory; CTA 0 writes
//      the routing outputs and the histogram
//   C  gate/up + SwiGLU: each CTA owns a contiguous range of 16-row tiles of
//      the selected experts; codes and scales stream through a ring of TMA
//      stages; the dot products run on mma.sync m16n8k16 (bf16 in, fp32 out)
//      with all T tokens as the 8 columns, so the cost per weight is the
//      unpack alone; W_d rows needed in D are prefetched into L2
//   -- barrier --
//   D  down + combine: each CTA owns 16 output features for every selected
//      expert, so it holds complete sums and writes out[t][f] directly, in
//      a fixed slot order.
//
// Codes enter the MMA as (128 + q) in bf16 (an exponent-bias bit pattern:
// 0x4300 | q), so each block's MMA result is sum q x + 128 sum x; the block
// correction (128 + offset) * sum x is subtracted and the block scale applied
// in fp32.  All waits (ring mbarriers, grid barriers) are bounded.
#pragma once
#include "common.cuh"
#include "perm.cuh"
#include "router.cuh"

#define DF_WARPS 16
#define DF_THREADS (32 * DF_WARPS)
#define DF_STAGES 12     // ring slots: DF_GROUPS private rings of DF_GSLOTS
#define DF_GSLOTS 4
#define DF_SLOT 10240    // 10 KB, a multiple of 1024 (swizzled boxes)
#define DF_HSTAGE 4      // pairs whose h is staged with a phase-D unit
#define DF_GROUPS 3      // consumer groups
#define DF_GW 4          // warps per consumer group (warps 1..12)
#define DF_BPW 4         // quant blocks per warp in a phase-C unit (DF_CHUNK / 32 / DF_GW)
#define DF_CHUNK 512     // gate/up K-chunk staged per ring unit
#define DF_TN 8          // token columns of the MMA
#define DF_MAXP 256      // pairs T * k
#define DF_FT 16         // features per CTA in phase D

struct DecodeFusedArgs {
    const uint8_t* arena;
    const int32_t* slot_table;
    int64_t n_slots;
    int64_t off_codes[3], off_scales[3];
    int64_t slot_bytes;
    int H, I, E, k, layer, T, residual;
    int bits_g, bits_u, bits_d;
    const uint16_t* x;       // [T][H]
    const float* W;          // router [E][H]
    const float* b;          // router bias [E] or null
    uint16_t* out;           // [T][H]
    uint32_t* hist;          // [L][E] or null
    int32_t* idx;            // [T*k]
    float* w;                // [T*k]
    int32_t* offsets;        // [E+1]
    int32_t* perm;           // [T*k]
    int32_t* nrechk;         // [1]
    double* logit;           // [T][E] workspace
    double* absum;           // [T][E] workspace (unused by the fused kernel)
    float* wnorm;            // [E] upper bounds of ||W[e]||_2 (workspace)
    uint16_t* hB;            // [P][I] bf16, MMA-fragment order within each 32-block
    float* hC;               // [P][I/16] sums of h over 16-row halves of each block
    unsigned int* bar;       // grid barrier counter (zeroed before launch)
};

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier over `nblocks` co-resident CTAs; the counter only grows
// (target = nblocks * phase).  Bounded: on expiry the status word gets
// MOE_ERR_TIMEOUT and every thread of the CTA sees false.
__device__ __forceinline__ bool grid_barrier(unsigned* ctr, unsigned target, int site) {
    __syncthreads();
    int ok = 1;
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
        unsigned it = 0;
        while (ld_acquire_u32(ctr) < target) {
            if (++it > MOE_SPIN_LIMIT) { moe_note_timeout(site, (int)(ld_acquire_u32(ctr) % 1000)); ok = 0; break; }
            if (it > 32) __nanosleep(64);
        }
        __threadfence();
    }
    return __syncthreads_and(ok) != 0;
}

// Barrier among the 4 warps of consumer group gr (named barriers 1..3).
__device__ __forceinline__ void group_sync(int gr) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + gr), "r"(32 * DF_GW) : "memory");
}

// The same barrier, returning whether `ok` holds in every thread of the group,
// so the group takes one decision (all of its warps keep meeting the barrier).
__device__ __forceinline__ bool group_sync_and(int gr, bool ok) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred pin, pout;\n setp.ne.u32 pin, %1, 0;\n bar.red.and.pred pout, %2, %3, pin;\n"
        " selp.u32 %0, 1, 0, pout;\n}"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(1 + gr), "r"(32 * DF_GW)
        : "memory");
    return r != 0;
}

// bf16 pairs (128 + q_i, 128 + q_{i+4}) of 8 codes: 4-bit word w = codes
// 0..7 in nibbles; 2-bit: codes 0..7 in the low 16 bits.
template <int BITS>
__device__ __forceinline__ void unpack8(uint32_t w, uint32_t (&p)[4]) {
    if (BITS == 4) {
        p[0] = (w & 0x000F000Fu) | 0x43004300u;
        p[1] = ((w >> 4) & 0x000F000Fu) | 0x43004300u;
        p[2] = ((w >> 8) & 0x000F000Fu) | 0x43004300u;
        p[3] = ((w >> 12) & 0x000F000Fu) | 0x43004300u;
    } else {
        const uint32_t v = __byte_perm(w, 0, 0x4140);  // byte0 -> byte 0, byte1 -> byte 2
        p[0] = (v & 0x00030003u) | 0x43004300u;
        p[1] = ((v >> 2) & 0x00030003u) | 0x43004300u;
        p[2] = ((v >> 4) & 0x00030003u) | 0x43004300u;
        p[3] = ((v >> 6) & 0x00030003u) | 0x43004300u;
    }
}

// D(4 fp32) += A(16x16 bf16) * B(16x8 bf16)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of thread q's 8 codes of quant block c (within its 128-byte box
// row) for a row whose swizzle key is key16 = (row & 7) << 4: the TMA 128-byte
// swizzle XORs the 16-byte chunk index with the row's low 3 bits.
template <int BITS>
__device__ __forceinline__ int sw_off(int c, int q, int key16) {
    constexpr int BLK_B = 32 * BITS / 8;  // bytes per quant block
    const int off = c * BLK_B + q * BITS;
    return ((off & ~15) ^ key16) | (off & 15);
}

template <int BITS>
__device__ __forceinline__ uint32_t ld_codes(const uint8_t* p) {
    if (BITS == 4) return *reinterpret_cast<const uint32_t*>(p);
    return *reinterpret_cast<const uint16_t*>(p);
}

// 8 bf16 of a row in the fragment order used for B: elements (0,4),(1,5),(2,6),(3,7)
__device__ __forceinline__ uint4 frag_order8(const float (&v)[8]) {
    uint4 r;
    r.x = pack_bf16x2(v[0], v[4]);
    r.y = pack_bf16x2(v[1], v[5]);
    r.z = pack_bf16x2(v[2], v[6]);
    r.w = pack_bf16x2(v[3], v[7]);
    return r;
}

// ---------------------------------------------------------------- shared memory plan

struct DfRoute {  // grouping of the window's pairs, identical in every CTA
    int32_t idx[DF_MAXP];   // expert of pair p = t*k + j
    float w[DF_MAXP];
    int32_t perm[DF_MAXP];  // position -> pair
    int32_t inv[DF_MAXP];   // pair -> position
    int32_t u_e[DF_MAXP];   // selected experts, ascending
    int32_t u_pos[DF_MAXP]; // first position of each
    int32_t u_n[DF_MAXP];   // pairs of each
    int32_t n_uniq;
};

// ---------------------------------------------------------------- phase C: one 16-row tile, one K-chunk

// Ring unit of phase C: [gate code boxes][up code boxes][gate scales 16 x 16][up scales 16 x 16].
// Accumulates gate and up for rows (g, g+8) of the tile and token columns
// (2q, 2q+1).  The block correction enters as the MMA's C input: xcg/xcu hold
// -(128 + offset) * sum x per (block, token).
template <int BG, int BU>
__device__ __forceinline__ void gateup_chunk(const uint8_t* slot, int nbox_g, int nbox_u, int j0, int jb,
                                             const uint4* xb, const float* xcg, const float* xcu, float (&accg)[4],
                                             float (&accu)[4]) {
    constexpr int NBLK = DF_CHUNK / 32;
    constexpr int PG = 128 / (32 * BG / 8), PU = 128 / (32 * BU / 8);  // quant blocks per 128-byte box row
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, key16 = (g & 7) << 4;
    const uint8_t* cg0 = slot + g * 128;
    const uint8_t* cg1 = cg0 + 8 * 128;
    const uint8_t* cu0 = slot + nbox_g * 2048 + g * 128;
    const uint8_t* cu1 = cu0 + 8 * 128;
    const uint16_t* sg = reinterpret_cast<const uint16_t*>(slot + (nbox_g + nbox_u) * 2048);
    const uint16_t* su = sg + 16 * NBLK;
#pragma unroll
    for (int jj = jb; jj < jb + DF_BPW; jj += 2) {  // this warp's quant blocks of the chunk
        const float2 fg0 = __half22float2(*reinterpret_cast<const __half2*>(sg + g * NBLK + jj));
        const float2 fg1 = __half22float2(*reinterpret_cast<const __half2*>(sg + (g + 8) * NBLK + jj));
        const float2 fu0 = __half22float2(*reinterpret_cast<const __half2*>(su + g * NBLK + jj));
        const float2 fu1 = __half22float2(*reinterpret_cast<const __half2*>(su + (g + 8) * NBLK + jj));
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int j = jj + h2;
            const uint4 bx = xb[((j0 + j) * 4 + q) * DF_TN + g];
            const float2 cgv = *reinterpret_cast<const float2*>(xcg + (j0 + j) * DF_TN + 2 * q);
            const float2 cuv = *reinterpret_cast<const float2*>(xcu + (j0 + j) * DF_TN + 2 * q);
            const int og = (j / PG) * 2048 + sw_off<BG>(j % PG, q, key16);
            const int ou = (j / PU) * 2048 + sw_off<BU>(j % PU, q, key16);
            uint32_t pg0[4], pg1[4], pu0[4], pu1[4];
            unpack8<BG>(ld_codes<BG>(cg0 + og), pg0);
            unpack8<BG>(ld_codes<BG>(cg1 + og), pg1);
            unpack8<BU>(ld_codes<BU>(cu0 + ou), pu0);
            unpack8<BU>(ld_codes<BU>(cu1 + ou), pu1);
            float dg[4] = {cgv.x, cgv.y, cgv.x, cgv.y}, du[4] = {cuv.x, cuv.y, cuv.x, cuv.y};
            mma_bf16_16816(dg, pg0[0], pg1[0], pg0[1], pg1[1], bx.x, bx.y);
            mma_bf16_16816(dg, pg0[2], pg1[2], pg0[3], pg1[3], bx.z, bx.w);
            mma_bf16_16816(du, pu0[0], pu1[0], pu0[1], pu1[1], bx.x, bx.y);
            mma_bf16_16816(du, pu0[2], pu1[2], pu0[3], pu1[3], bx.z, bx.w);
            const float sg0 = h2 ? fg0.y : fg0.x, sg1 = h2 ? fg1.y : fg1.x;
            const float su0 = h2 ? fu0.y : fu0.x, su1 = h2 ? fu1.y : fu1.x;
            accg[0] = fmaf(sg0, dg[0], accg[0]);
            accg[1] = fmaf(sg0, dg[1], accg[1]);
            accg[2] = fmaf(sg1, dg[2], accg[2]);
            accg[3] = fmaf(sg1, dg[3], accg[3]);
            accu[0] = fmaf(su0, du[0], accu[0]);
            accu[1] = fmaf(su0, du[1], accu[1]);
            accu[2] = fmaf(su1, du[2], accu[2]);
            accu[3] = fmaf(su1, du[3], accu[3]);
        }
    }
}

// ---------------------------------------------------------------- phase D: one expert's 16 features

// Ring unit of phase D: [W_d code boxes][scales 16 x I/32][h of the expert's n
// pairs, bf16 fragment order][sums of h over 16-row halves].  Column g of B is
// pair g of the expert (zero when g >= n).
template <int BD>
__device__ __forceinline__ void down_unit(const uint8_t* slot, int nbox, int I, int n, const uint16_t* hB_g,
                                          const float* hC_g, int jbeg, int jend, float (&acc)[4]) {
    constexpr int PB = 128 / (32 * BD / 8);
    constexpr float kOff = 128.f + (float)(1 << (BD - 1));
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, key16 = (g & 7) << 4;
    const int nblk = I / 32;
    const uint8_t* c0 = slot + g * 128;
    const uint8_t* c1 = c0 + 8 * 128;
    const uint16_t* sd = reinterpret_cast<const uint16_t*>(slot + nbox * 2048);
    const int ns = min(n, DF_HSTAGE);  // pairs staged in the slot; the rest are read from L2
    const uint4* hbs = reinterpret_cast<const uint4*>(slot + nbox * 2048 + 16 * nblk * 2);
    const float* hcs = reinterpret_cast<const float*>(slot + nbox * 2048 + 16 * nblk * 2 + ns * I * 2);
    const bool col_ok = g < n, ok0 = 2 * q < n, ok1 = 2 * q + 1 < n;
    const uint4* hb = g < ns ? hbs + (size_t)g * nblk * 4 : reinterpret_cast<const uint4*>(hB_g) + (size_t)g * nblk * 4;
    const float* hc0 = 2 * q < ns ? hcs + (2 * q) * (I / 16) : hC_g + (2 * q) * (I / 16);
    const float* hc1 = 2 * q + 1 < ns ? hcs + (2 * q + 1) * (I / 16) : hC_g + (2 * q + 1) * (I / 16);
#pragma unroll 4
    for (int j = jbeg; j < jend; ++j) {
        const uint4 bx = col_ok ? hb[j * 4 + q] : make_uint4(0, 0, 0, 0);
        const float h0 = ok0 ? hc0[2 * j] + hc0[2 * j + 1] : 0.f;
        const float h1 = ok1 ? hc1[2 * j] + hc1[2 * j + 1] : 0.f;
        const int o = (j / PB) * 2048 + sw_off<BD>(j % PB, q, key16);
        uint32_t p0[4], p1[4];
        unpack8<BD>(ld_codes<BD>(c0 + o), p0);
        unpack8<BD>(ld_codes<BD>(c1 + o), p1);
        float d[4] = {-kOff * h0, -kOff * h1, -kOff * h0, -kOff * h1};
        mma_bf16_16816(d, p0[0], p1[0], p0[1], p1[1], bx.x, bx.y);
        mma_bf16_16816(d, p0[2], p1[2], p0[3], p1[3], bx.z, bx.w);
        const float s0 = half_bits_to_f32(sd[g * nblk + j]), s1 = half_bits_to_f32(sd[(g + 8) * nblk + j]);
        acc[0] = fmaf(s0, d[0], acc[0]);
        acc[1] = fmaf(s0, d[1], acc[1]);
        acc[2] = fmaf(s1, d[2], acc[2]);
        acc[3] = fmaf(s1, d[3], acc[3]);
    }
}

// ---------------------------------------------------------------- the kernel

__host__ __device__ constexpr int df_smem_bytes(int H) {
    return 1024 /*align*/ + DF_STAGES * DF_SLOT + H * 16 /*x fragments*/ + 2 * (H / 32) * DF_TN * 4 /*corrections*/ +
           DF_MAXP * DF_FT * 4 /*per-pair outputs*/ + DF_GROUPS * DF_GW * 32 * 8 * 4 /*group partials*/ +
           (int)sizeof(DfRoute) + 2 * DF_STAGES * 8 + 64;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

template <int BG, int BU, int BD>
__global__ void __launch_bounds__(DF_THREADS, 1)
    k_decode_fused(const __grid_constant__ CUtensorMap tcg, const __grid_constant__ CUtensorMap tcu,
                   const __grid_constant__ CUtensorMap tcd, const __grid_constant__ CUtensorMap tsg,
                   const __grid_constant__ CUtensorMap tsu, const __grid_constant__ CUtensorMap tsd,
                   DecodeFusedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int H = a.H, I = a.I, E = a.E, k = a.k, T = a.T, P = T * k, NB = H / 32;
    uint4* xb = reinterpret_cast<uint4*>(ring + DF_STAGES * DF_SLOT);  // [NB][4][8] x fragments
    float* xcg = reinterpret_cast<float*>(xb + NB * 4 * DF_TN);        // [NB][8] -(128+off_g) sum x
    float* xcu = xcg + NB * DF_TN;                                       // [NB][8] -(128+off_u) sum x
    float* xpart = reinterpret_cast<float*>(ring);                      // [NB][4][8] partial sums (ring is idle)
    float* ypair = xcu + NB * DF_TN;                                     // [MAXP][FT]
    DfRoute* rt = reinterpret_cast<DfRoute*>(ypair + DF_MAXP * DF_FT + DF_GROUPS * DF_GW * 32 * 8);
    uint64_t* full = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(rt + 1) + 7) & ~(uintptr_t)7);
    uint64_t* empty = full + DF_STAGES;
    __shared__ int s_cnt[MOE_MAX_E];
    __shared__ int s_off[MOE_MAX_E];
    __shared__ int s_warp[33];
    __shared__ float s_xnorm[DF_TN];

    const int G = gridDim.x, cta = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    bool alive = true;

    if (tid == 0) {
        for (int s = 0; s < DF_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], DF_GW);  // every warp of the consuming group releases the unit
        }
        fence_mbar_init();
    }

    // ---- A: router logits in fp64 on the tensor cores (mma.m8n8k4.f64).  A CTA
    // takes experts 8o..8o+7; its warps split H.  Every bf16 x fp32 product is
    // exact in fp64, so only the additions round (bound: gamma_(H+32)).
    for (int oc = cta; oc * 8 < E; oc += G) {
        const int e0 = oc * 8, g = lane >> 2, q = lane & 3, eg = e0 + g;
        const int kw = H / DF_WARPS, kb = warp * kw;
        const float* wrow = a.W + (size_t)min(eg, E - 1) * H;
        const uint16_t* xrow = a.x + (size_t)min(g, T - 1) * H;
        double c0 = 0.0, c1 = 0.0;
        float w2 = 0.f;
#pragma unroll 4
        for (int k0 = kb; k0 < kb + kw; k0 += 16) {
            // step s of this 16-element slice uses k = k0 + 4 q + s (A and B alike)
            const float4 wv = eg < E ? __ldg(reinterpret_cast<const float4*>(wrow + k0 + 4 * q)) : make_float4(0, 0, 0, 0);
            const uint2 xv = g < T ? __ldg(reinterpret_cast<const uint2*>(xrow + k0 + 4 * q)) : make_uint2(0, 0);
            w2 = fmaf(wv.x, wv.x, fmaf(wv.y, wv.y, fmaf(wv.z, wv.z, fmaf(wv.w, wv.w, w2))));
            const double av[4] = {wv.x, wv.y, wv.z, wv.w};
            const double bv[4] = {__uint_as_float(xv.x << 16), __uint_as_float(xv.x & 0xffff0000u),
                                  __uint_as_float(xv.y << 16), __uint_as_float(xv.y & 0xffff0000u)};
#pragma unroll
            for (int st = 0; st < 4; ++st)
                asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                             : "+d"(c0), "+d"(c1)
                             : "d"(av[st]), "d"(bv[st]));
        }
        // c0, c1: expert eg, tokens 2q, 2q+1 (this warp's slice of H)
        double* sp = reinterpret_cast<double*>(ring);  // the ring is free during A
        sp[(warp * 8 + g) * 8 + 2 * q] = c0;
        sp[(warp * 8 + g) * 8 + 2 * q + 1] = c1;
        w2 += __shfl_xor_sync(0xffffffffu, w2, 1);
        w2 += __shfl_xor_sync(0xffffffffu, w2, 2);
        float* sw2 = reinterpret_cast<float*>(ring + DF_WARPS * 64 * 8);
        if (q == 0) sw2[warp * 8 + g] = w2;
        __syncthreads();
        if (tid < 64) {
            const int gg = tid >> 3, t = tid & 7, e = e0 + gg;
            if (e < E && t < T) {
                double sum = 0.0;
                for (int w = 0; w < DF_WARPS; ++w) sum += sp[(w * 8 + gg) * 8 + t];
                a.logit[(size_t)t * E + e] = sum + (a.b ? (double)a.b[e] : 0.0);
            }
        } else if (tid < 72) {
            const int e = e0 + tid - 64;
            if (e < E) {
                float s2 = 0.f;
                for (int w = 0; w < DF_WARPS; ++w) s2 += sw2[w * 8 + tid - 64];
                a.wnorm[e] = sqrtf(s2) * 1.001f;
            }
        }
        __syncthreads();
    }

    // x as MMA B fragments (token columns 0..7, zero beyond T) and block corrections
    for (int u = tid; u < NB * 4 * DF_TN; u += DF_THREADS) {
        const int n = u % DF_TN, q = (u / DF_TN) % 4, j = u / (DF_TN * 4);
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (n < T) {
            uint4 r4 = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)n * H + 32 * j + 8 * q));
            v[0] = __uint_as_float(r4.x << 16); v[1] = __uint_as_float(r4.x & 0xffff0000u);
            v[2] = __uint_as_float(r4.y << 16); v[3] = __uint_as_float(r4.y & 0xffff0000u);
            v[4] = __uint_as_float(r4.z << 16); v[5] = __uint_as_float(r4.z & 0xffff0000u);
            v[6] = __uint_as_float(r4.w << 16); v[7] = __uint_as_float(r4.w & 0xffff0000u);
        }
        xb[u] = frag_order8(v);
        xpart[u] = ((((((v[0] + v[1]) + v[2]) + v[3]) + v[4]) + v[5]) + v[6]) + v[7];
        float sq = 0.f;
#pragma unroll
        for (int z = 0; z < 8; ++z) sq = fmaf(v[z], v[z], sq);
        xpart[NB * 4 * DF_TN + u] = sq;
    }
    __syncthreads();
    if (warp < T) {  // ||x_t|| for the top-k bounds (inflated over its fp32 rounding)
        float sq = 0.f;
        for (int u = lane; u < NB * 4; u += 32) sq += xpart[NB * 4 * DF_TN + u * DF_TN + warp];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_xnorm[warp] = sqrtf(sq) * 1.001f;
    }
    for (int u = tid; u < NB * DF_TN; u += DF_THREADS) {
        const int n = u % DF_TN, j = u / DF_TN;
        const float* pp = xpart + (size_t)j * 4 * DF_TN + n;
        const float sx = ((pp[0] + pp[DF_TN]) + pp[2 * DF_TN]) + pp[3 * DF_TN];
        xcg[u] = -(128.f + (float)(1 << (BG - 1))) * sx;
        xcu[u] = -(128.f + (float)(1 << (BU - 1))) * sx;
    }
    alive = grid_barrier(a.bar, (unsigned)G, 1);  // uniform across the CTA

    // ---- B: certified top-k of every token (same result in every CTA) and grouping
    if (alive) {
        if (warp < T) {
            TopkArgs ta{};
            ta.x = a.x; ta.W = a.W; ta.b = a.b; ta.logit = a.logit; ta.wnorm = a.wnorm; ta.xnorm = s_xnorm;
            // phase-A sums: at most H + 32 roundings along any product's path
            ta.gfast = (double)(H + 32) * 1.1102230246251565e-16 * 1.01;
            ta.T = T; ta.H = H; ta.E = E; ta.k = k;
            int* cs = reinterpret_cast<int*>(ring) + warp * MOE_MAX_E;  // the ring is free during B
            double* cvs = reinterpret_cast<double*>(ring + DF_TN * MOE_MAX_E * 4) + warp * MOE_MAX_E;
            topk_token<2>(ta, warp, rt->idx + warp * k, rt->w + warp * k, cs, cvs, cta == 0 ? a.nrechk : nullptr);
        }
        for (int e = tid; e < MOE_MAX_E; e += DF_THREADS) s_cnt[e] = 0;
        __syncthreads();
        for (int p = tid; p < P; p += DF_THREADS) atomicAdd(&s_cnt[rt->idx[p]], 1);
        __syncthreads();
        const int c = tid < E ? s_cnt[tid] : 0;
        int off;
        const int total = block_excl_scan(c, &off, s_warp);
        if (tid < E) s_off[tid] = off;
        int upos;
        const int nu = block_excl_scan((tid < E && c > 0) ? 1 : 0, &upos, s_warp);
        if (tid < E && c > 0) {
            rt->u_e[upos] = tid;
            rt->u_pos[upos] = off;
            rt->u_n[upos] = c;
        }
        if (tid == 0) rt->n_uniq = nu;
        if (cta == 0) {
            if (tid < E) {
                a.offsets[tid] = off;
                if (a.hist) a.hist[(size_t)a.layer * E + tid] += (uint32_t)c;
                if (c > 0) {
                    const int64_t sl = a.slot_table[(int64_t)a.layer * E + tid];
                    if (sl < 0 || sl >= a.n_slots) moe_set_status(MOE_ERR_SLOT);
                }
            }
            if (tid == 0) a.offsets[E] = total;
        }
        __syncthreads();
        for (int p = tid; p < P; p += DF_THREADS) {
            const int e = rt->idx[p];
            int before = 0;
            for (int q2 = 0; q2 < p; ++q2) before += (rt->idx[q2] == e);
            const int pos = s_off[e] + before;
            rt->perm[pos] = p;
            rt->inv[p] = pos;
            if (cta == 0) {
                a.perm[pos] = p;
                a.idx[p] = e;
                a.w[p] = rt->w[p];
            }
        }
        __syncthreads();
    }

    // ---- C: gate/up + SwiGLU over this CTA's range of 16-row tiles.  Three groups
    // of 4 consumer warps; group gr owns tiles gr, gr+3, ...; the 4 warps of a
    // group split the 16 quant blocks of every unit and combine at the tile end.
    const int tiles_per_e = I / 16;
    const int nuq = alive ? rt->n_uniq : 0;
    const int R = nuq * tiles_per_e;
    const int r0 = (int)((int64_t)cta * R / G), r1 = (int)((int64_t)(cta + 1) * R / G);
    const int nloc = r1 - r0;
    const int nch = H / DF_CHUNK;
    constexpr int nbox_g = DF_CHUNK * BG / 8 / 128, nbox_u = DF_CHUNK * BU / 8 / 128;
    constexpr uint32_t bytes_c = (uint32_t)((nbox_g + nbox_u) * 2048 + 2 * 16 * (DF_CHUNK / 32) * 2);
    int Sc[DF_GROUPS];  // units of each group in phase C
#pragma unroll
    for (int gr = 0; gr < DF_GROUPS; ++gr) Sc[gr] = (nloc > gr ? (nloc - gr + DF_GROUPS - 1) / DF_GROUPS : 0) * nch;
    const int ft0 = cta * DF_FT;  // phase-D features of this CTA
    const int rowb_d = I * BD / 8;
    const int grp = (warp - 1) / DF_GW, gw = (warp - 1) % DF_GW;  // consumer group and rank (warps 1..12)
    const bool consumer = warp >= 1 && warp <= DF_GROUPS * DF_GW;
    float* gpart = reinterpret_cast<float*>(ypair + DF_MAXP * DF_FT);  // [group][warp][lane][8] partial sums

    // Everything this CTA will read in C and D goes to L2 at once: HBM then
    // streams at full rate whatever the shared-memory ring can hold, and the
    // ring refills from L2.  Gate/up tiles first (16 contiguous rows each),
    // then the W_d rows of this CTA's features for every selected expert.
    if (alive) {
        const int rowb_g = H * BG / 8, rowb_u = H * BU / 8;
        for (int lt = tid; lt < nloc; lt += DF_THREADS) {
            const int gt = r0 + lt, ui = gt / tiles_per_e, r16 = gt % tiles_per_e;
            const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
            if (sl < 0 || sl >= a.n_slots) continue;
            const uint8_t* base = a.arena + sl * a.slot_bytes;
            prefetch_l2(base + a.off_codes[0] + (int64_t)r16 * 16 * rowb_g, (uint32_t)(16 * rowb_g));
            prefetch_l2(base + a.off_codes[1] + (int64_t)r16 * 16 * rowb_u, (uint32_t)(16 * rowb_u));
            prefetch_l2(base + a.off_scales[0] + (int64_t)r16 * 16 * (H / 16), (uint32_t)(16 * (H / 16)));
            prefetch_l2(base + a.off_scales[1] + (int64_t)r16 * 16 * (H / 16), (uint32_t)(16 * (H / 16)));
        }
        if (ft0 < H)
            for (int ft = ft0; ft < H; ft += G * DF_FT)
                for (int ui = tid; ui < nuq; ui += DF_THREADS) {
                    const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                    if (sl < 0 || sl >= a.n_slots) continue;
                    const uint8_t* base = a.arena + sl * a.slot_bytes;
                    prefetch_l2(base + a.off_codes[2] + (int64_t)ft * rowb_d, (uint32_t)(DF_FT * rowb_d));
                    prefetch_l2(base + a.off_scales[2] + (int64_t)ft * (I / 32) * 2, (uint32_t)(DF_FT * (I / 32) * 2));
                }
    }

    const bool producer = warp >= DF_WARPS - DF_GROUPS;  // warps 13..15 feed groups 0..2
    if (producer) {
        const int gr = warp - (DF_WARPS - DF_GROUPS);
        if (lane == 0 && alive) {
            fence_proxy_async_smem();  // the ring held generic-proxy scratch during A and B
            for (int st = 0; st < Sc[gr]; ++st) {
                const int lt = gr + DF_GROUPS * (st / nch), ch = st % nch;
                const int gt = r0 + lt, ui = gt / tiles_per_e, r16 = gt % tiles_per_e;
                const int s = gr * DF_GSLOTS + st % DF_GSLOTS, ph = (st / DF_GSLOTS) & 1;
                const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                if (!mbar_wait(&empty[s], ph ^ 1, 3, st)) break;
                uint8_t* dst = ring + s * DF_SLOT;
                if (sl < 0 || sl >= a.n_slots) {  // nothing to load: release the consumers
                    mbar_arrive(&full[s]);
                    continue;
                }
                mbar_arrive_expect_tx(&full[s], bytes_c);
#pragma unroll
                for (int bx = 0; bx < nbox_g; ++bx)
                    tma_load_3d(dst + bx * 2048, &tcg, &full[s], ch * DF_CHUNK * BG / 8 + bx * 128, r16 * 16, (int)sl);
#pragma unroll
                for (int bx = 0; bx < nbox_u; ++bx)
                    tma_load_3d(dst + (nbox_g + bx) * 2048, &tcu, &full[s], ch * DF_CHUNK * BU / 8 + bx * 128, r16 * 16,
                                (int)sl);
                uint8_t* sdst = dst + (nbox_g + nbox_u) * 2048;
                tma_load_3d(sdst, &tsg, &full[s], ch * DF_CHUNK / 32, r16 * 16, (int)sl);
                tma_load_3d(sdst + 16 * (DF_CHUNK / 32) * 2, &tsu, &full[s], ch * DF_CHUNK / 32, r16 * 16, (int)sl);
            }
        }
    } else if (consumer && alive) {
        const int g = lane >> 2, q = lane & 3;
        float* mypart = gpart + ((grp * DF_GW + gw) * 32 + lane) * 8;
        for (int st0 = 0; st0 < Sc[grp] && alive; st0 += nch) {
            const int lt = grp + DF_GROUPS * (st0 / nch);
            const int gt = r0 + lt, ui = gt / tiles_per_e, r16 = gt % tiles_per_e;
            const int e = rt->u_e[ui], pos0 = rt->u_pos[ui], n = rt->u_n[ui];
            const int64_t sl = a.slot_table[(int64_t)a.layer * E + e];
            const bool valid = sl >= 0 && sl < a.n_slots;
            float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
            bool ok = true;
            for (int ch = 0; ch < nch && ok; ++ch) {
                const int st = st0 + ch;  // unit index in this group's ring
                const int s = grp * DF_GSLOTS + st % DF_GSLOTS, ph = (st / DF_GSLOTS) & 1;
                ok = mbar_wait(&full[s], ph, 4, st);
                if (ok && valid)
                    gateup_chunk<BG, BU>(ring + s * DF_SLOT, nbox_g, nbox_u, ch * (DF_CHUNK / 32), gw * DF_BPW, xb, xcg,
                                         xcu, accg, accu);
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&empty[s]);
            }
            // combine the group's 4 partial sums (fixed order), then h for every pair of the expert
#pragma unroll
            for (int z = 0; z < 4; ++z) { mypart[z] = accg[z]; mypart[4 + z] = accu[z]; }
            if (!group_sync_and(grp, ok)) { alive = false; break; }  // the whole group leaves together
            if (gw == 0) {
#pragma unroll
                for (int w2 = 1; w2 < DF_GW; ++w2) {
                    const float* op = gpart + ((grp * DF_GW + w2) * 32 + lane) * 8;
#pragma unroll
                    for (int z = 0; z < 4; ++z) { accg[z] += op[z]; accu[z] += op[4 + z]; }
                }
                for (int jj = 0; jj < n; ++jj) {
                    const int pos = pos0 + jj, t = rt->perm[pos] / k;
                    const bool mine = (t >> 1) == q;
                    const int sel = t & 1;
                    float h0 = 0.f, h1 = 0.f;  // rows g, g + 8
                    if (mine && valid) {
                        h0 = silu_f32(sel ? accg[1] : accg[0]) * (sel ? accu[1] : accu[0]);
                        h1 = silu_f32(sel ? accg[3] : accg[2]) * (sel ? accu[3] : accu[2]);
                    }
                    const uint16_t b0 = f32_to_bf16_bits(h0), b1 = f32_to_bf16_bits(h1);
                    float part = bf16_bits_to_f32(b0) + bf16_bits_to_f32(b1);
                    part += __shfl_xor_sync(0xffffffffu, part, 4);
                    part += __shfl_xor_sync(0xffffffffu, part, 8);
                    part += __shfl_xor_sync(0xffffffffu, part, 16);
                    if (mine) {
                        // element rr of I lands at block rr/32, quad (rr%32)/8, fragment slot of rr%8
                        const int rows[2] = {r16 * 16 + g, r16 * 16 + g + 8};
                        const uint16_t vals[2] = {b0, b1};
#pragma unroll
                        for (int z = 0; z < 2; ++z) {
                            const int rr = rows[z], e32 = rr & 31, i8 = e32 & 7;
                            a.hB[(size_t)pos * I + (rr & ~31) + (e32 >> 3) * 8 + (i8 & 3) * 2 + (i8 >> 2)] = vals[z];
                        }
                        if (g == 0) a.hC[(size_t)pos * (I / 16) + r16] = part;
                    }
                }
            }
            group_sync(grp);  // partial buffer free for the next tile
        }
        fence_proxy_async_global();  // h is read back by bulk copies after the barrier
    }
    {
        const int mine_ok = alive ? 1 : 0;
        const bool gb = grid_barrier(a.bar, 2u * (unsigned)G, 2);
        alive = __syncthreads_and(mine_ok && gb) != 0;
    }

    // ---- D: down projection for this CTA's feature tiles (16 features each), every
    // selected expert (group gr takes experts gr, gr+3, ...); then the combine.
    if (alive) {
        const int nbox_d = rowb_d / 128;
        const int sc_d = 16 * (I / 32) * 2;  // scale bytes of a unit
        const int nblk_d = I / 32, bpw_d = (nblk_d + DF_GW - 1) / DF_GW;
        int Sd[DF_GROUPS];
#pragma unroll
        for (int gr = 0; gr < DF_GROUPS; ++gr) Sd[gr] = nuq > gr ? (nuq - gr + DF_GROUPS - 1) / DF_GROUPS : 0;
        int rnd = 0;  // feature-tile round; each group's ring units continue from phase C
        for (int ft = ft0; ft < H; ft += G * DF_FT, ++rnd) {
            if (producer) {
                const int gr = warp - (DF_WARPS - DF_GROUPS);
                if (lane == 0) {
                    fence_proxy_async_global();
                    for (int st = 0; st < Sd[gr]; ++st) {
                        const int ui = gr + DF_GROUPS * st, u = Sc[gr] + rnd * Sd[gr] + st;
                        const int s = gr * DF_GSLOTS + u % DF_GSLOTS, ph = (u / DF_GSLOTS) & 1;
                        const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                        const int n = rt->u_n[ui], pos0 = rt->u_pos[ui];
                        if (!mbar_wait(&empty[s], ph ^ 1, 5, u)) break;
                        uint8_t* dst = ring + s * DF_SLOT;
                        if (sl < 0 || sl >= a.n_slots) {
                            mbar_arrive(&full[s]);
                            continue;
                        }
                        const int ns = min(n, DF_HSTAGE);  // pairs staged in the unit
                        const uint32_t hbytes = (uint32_t)(ns * I * 2), cbytes = (uint32_t)(ns * (I / 16) * 4);
                        mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox_d * 2048 + sc_d) + hbytes + cbytes);
                        for (int bx = 0; bx < nbox_d; ++bx)
                            tma_load_3d(dst + bx * 2048, &tcd, &full[s], bx * 128, ft, (int)sl);
                        tma_load_3d(dst + nbox_d * 2048, &tsd, &full[s], 0, ft, (int)sl);
                        bulk_load(dst + nbox_d * 2048 + sc_d, a.hB + (size_t)pos0 * I, hbytes, &full[s]);
                        bulk_load(dst + nbox_d * 2048 + sc_d + hbytes, a.hC + (size_t)pos0 * (I / 16), cbytes,
                                  &full[s]);
                    }
                }
            } else if (consumer) {
                const int g = lane >> 2, q = lane & 3;
                float* mypart = gpart + ((grp * DF_GW + gw) * 32 + lane) * 8;
                for (int st = 0; st < Sd[grp]; ++st) {
                    const int ui = grp + DF_GROUPS * st, u = Sc[grp] + rnd * Sd[grp] + st;
                    const int s = grp * DF_GSLOTS + u % DF_GSLOTS, ph = (u / DF_GSLOTS) & 1;
                    const int pos0 = rt->u_pos[ui], n = rt->u_n[ui];
                    const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                    const bool valid = sl >= 0 && sl < a.n_slots;
                    const bool ok = mbar_wait(&full[s], ph, 6, u);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    if (ok && valid)
                        down_unit<BD>(ring + s * DF_SLOT, nbox_d, I, n, a.hB + (size_t)pos0 * I,
                                      a.hC + (size_t)pos0 * (I / 16), gw * bpw_d, min(nblk_d, (gw + 1) * bpw_d), acc);
                    __syncwarp();
                    if (ok && lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
                    for (int z = 0; z < 4; ++z) mypart[z] = acc[z];
                    if (!group_sync_and(grp, ok)) break;  // the whole group leaves together
                    if (gw == 0) {
#pragma unroll
                        for (int w2 = 1; w2 < DF_GW; ++w2) {
                            const float* op = gpart + ((grp * DF_GW + w2) * 32 + lane) * 8;
#pragma unroll
                            for (int z = 0; z < 4; ++z) acc[z] += op[z];
                        }
                        // y for pair columns 2q, 2q+1 (when they exist), features g, g+8
#pragma unroll
                        for (int z = 0; z < 2; ++z) {
                            const int jj = 2 * q + z;
                            if (jj < n) {
                                const int pos = pos0 + jj;
                                const float wv = rt->w[rt->perm[pos]];
                                ypair[pos * DF_FT + g] = wv * acc[z];
                                ypair[pos * DF_FT + g + 8] = wv * acc[2 + z];
                            }
                        }
                    }
                    group_sync(grp);
                }
            }
            __syncthreads();
            for (int u = tid; u < T * DF_FT; u += DF_THREADS) {
                const int t = u / DF_FT, fl = u % DF_FT, f = ft + fl;
                float sum = 0.f;
                for (int j = 0; j < k; ++j) sum += ypair[rt->inv[t * k + j] * DF_FT + fl];
                if (a.residual) sum = bf16_bits_to_f32(a.x[(size_t)t * H + f]) + sum;
                a.out[(size_t)t * H + f] = f32_to_bf16_bits(sum);
            }
            __syncthreads();
        }
    }
}
