// Decode window (T <= 8 tokens) as one persistent, cooperatively launched
// kernel per layer: one CTA per SM, two grid-wide barriers.
//
//   A  router logits in fp64 on the tensor cores (mma.m8n8k4.f64): each CTA
//      takes a few experts; their W_r rows and the window's x arrive by bulk
//      copies into shared memory
//   -- barrier --
//   B  every CTA certifies the top-k of every token (the same deterministic
//      computation everywhere) and builds the grouping (pairs sorted by
//      expert) in shared memory; CTA 0 writes the routing outputs and the
//      histogram
//   C  gate/up + SwiGLU: each CTA owns a contiguous range of 16-row tiles of
//      the selected experts, cut into units of 16 rows x one 128-byte code
//      box per matrix.  Every warp owns a contiguous run of those units and
//      streams them itself through two private TMA slots (codes and scales,
//      issued by one lane): it waits for a unit, copies it into registers,
//      re-arms the slot with its next unit and only then computes, so both
//      slots of every warp are in flight almost all the time.  Partial tile
//      sums go to shared memory and are finished (SwiGLU, bf16 h) once the
//      CTA's warps are done.  A warp that runs out of C units already loads
//      its first W_d units.
//   -- barrier --
//   D  down + combine: each CTA owns 16 output features (a feature tile) for
//      every selected expert, so it holds complete sums and writes out[t][f]
//      directly, in a fixed slot order.  h of every pair is copied into
//      shared memory from L2; warps take experts round-robin with the same
//      two-slot streaming.
//
// The dot products run on mma.sync m16n8k16 (fp32 out) with the weights as A
// (16 rows) and the tokens (or an expert's pairs) as the 8 columns of B, so a
// weight costs its unpack and one lane-slot of an MMA.  Gate/up codes enter
// as fp16 (1024 + m q) (bit pattern 0x6400 | field, m = 1 or 16 by the
// code's bit position, see unpack8_f16) against x' / m, x' a per-token
// power-of-two multiple of x; W_d codes enter as bf16 (128 + q) (0x4300 | q)
// against h.  Each block's offset term enters as the MMA's C input and the
// block scale is applied in fp32.  All waits (mbarriers, grid barriers) are
// bounded.
#pragma once
#include "common.cuh"
#include "perm.cuh"
#include "router.cuh"

// Phase timestamps for measurement builds (-DMOE_PROBE): thread 0 of every
// CTA records the global timer at the phase boundaries.  Compiled out
// otherwise.
#ifdef MOE_PROBE
#define DF_WARPS_PROBE 16
__device__ unsigned long long g_df_probe[160][24];
#define DF_MARK(i)                                                                  \
    do {                                                                            \
        if (threadIdx.x == 0 && blockIdx.x < 160) {                                 \
            unsigned long long t_;                                                  \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                  \
            g_df_probe[blockIdx.x][i] = t_;                                         \
        }                                                                           \
    } while (0)
// per warp: cycles waiting for C units, computing them, the same for D, units of each
#define DF_NWP 10
__device__ unsigned long long g_df_wprobe[160][DF_WARPS_PROBE][DF_NWP];
#define DF_CLK(v) unsigned long long v = clock64()
#define DF_WACC(slot, val) \
    do { if ((threadIdx.x & 31) == 0 && blockIdx.x < 160) g_df_wprobe[blockIdx.x][threadIdx.x >> 5][slot] += (val); } while (0)
#else
#define DF_MARK(i) \
    do {           \
    } while (0)
#define DF_CLK(v) \
    do {          \
    } while (0)
#define DF_WACC(slot, val) \
    do {               \
    } while (0)
#endif

#define DF_WARPS 16
#define DF_THREADS (32 * DF_WARPS)
#define DF_NBUF 2          // TMA slots per warp
#define DF_CODE_SLOT 4096  // two code boxes of 16 rows x 128 B (128-byte swizzle)
#define DF_TN 8            // token columns of the MMA
#define DF_MAXP 256        // pairs T * k
#define DF_FT 16           // features per phase-D tile
#define DF_MAX_EPC 8       // router experts per CTA (rows of the fp64 MMA)
#define DF_MAX_NBD 16      // quant blocks of a W_d row (I <= 512)
#define DF_SMEM_LIMIT (227 * 1024)
#define DF_BAR_WORDS 32     // grid barrier: one counter on its own 128-byte line
#define DF_NREP 8          // copies of the (logit, bound) records that phase B reads
#define DF_CAND_BYTES 640  // phase-B candidate scratch of one token: 32 experts, 32 values + 32 bounds

// Shared-memory layout, computed on the host (df_plan) and passed in; offsets
// are from the 1024-byte aligned base of dynamic shared memory.
struct DfPlan {
    int sc_off, sc_slot;        // scale ring [DF_WARPS][DF_NBUF][sc_slot]
    int r1_off;                 // C: xb, xc, partials | D: h, hsum, ypair
    int xc_off, part_off, n_part, part_bytes;
    int hs_stride, hsum_off, ypair_off;
    int route_off, stab_off, bar_off, total;
    // phase A (code ring, free then): x rows, W_r rows, per-warp sums, x block sums
    int a_ws_off, a_sp_off, a_w2_off, a_xp_off;
    // phase B (code ring): the (logit, bound) records, their keys, per-token candidate
    // scratch (32 experts, 64 doubles), and the exact fallback's scratch: the token's
    // own record row when it is large enough (b_fb_off < 0), else a region of its own
    int b_rec_off, b_key_off, b_cand_off, b_fb_off, b_fb_stride;
};

struct DecodeFusedArgs {
    const uint8_t* arena;
    const int32_t* slot_table;
    int64_t n_slots;
    int64_t off_codes[3], off_scales[3];
    int64_t slot_bytes;
    int H, I, E, k, layer, T, residual;
    int bits_gate, bits_up, bits_down;
    int epc;                 // router experts per CTA
    const uint16_t* x;       // [T][H]
    const float* W;          // router [E][H]
    const float* b;          // router bias [E] or null
    uint16_t* out;           // [T][H]
    float* hout;             // [T][H] fp32 output rows before rounding (steering: a second kernel
                             // finishes them), or null: bf16 rows go straight to out
    uint32_t* hist;          // [L][E] or null
    int32_t* idx;            // [T*k]
    float* w;                // [T*k]
    int32_t* offsets;        // [E+1]
    int32_t* perm;           // [T*k]
    int32_t* nrechk;         // [1]
    double* logit;           // [T][E] workspace
    float* wnorm;            // [E] upper bounds of ||W[e]||_2 (workspace)
    double2* rec;            // [DF_NREP][T][E] (logit, error bound): CTA c reads copy c % DF_NREP
    uint2* reck;             // [DF_NREP][T][E] (key32 of the fp32 logit, upper end rounded up to fp32)
    uint16_t* hB;            // [P][I] bf16, MMA-fragment order within each 32-block
    unsigned int* bar;       // grid barrier counter, DF_BAR_WORDS words (zeroed before launch)
    unsigned spin_limit;     // polling bound of the grid barriers (MOE_SPIN_LIMIT; lowered only by a test)
    unsigned bar1_extra;     // 0; a test sets it to make grid barrier 1 unsatisfiable
    DfPlan pl;
};

__host__ __device__ inline int df_al(int v, int a) { return (v + a - 1) / a * a; }

// Codes per K-chunk of a gate/up unit: one 128-byte box row.
__host__ __device__ constexpr int df_ck(int bits) { return 1024 / bits; }

// Feature tiles of CTA c (tiles c, c + G, ...).
__host__ __device__ inline int df_nft(int c, int NFT, int G) { return c < NFT ? (NFT - 1 - c) / G + 1 : 0; }

// Upper bound of the 16-row gate/up tiles any CTA gets (an equal share).
__host__ inline int df_max_tiles(int P, int E, int I, int G) {
    const int nuq = std::min(P, E);
    return (nuq * (I / 16) + G - 1) / G + 1;
}

// Returns false when the window does not fit one CTA's shared memory.
__host__ inline bool df_plan(DfPlan& p, int T, int P, int E, int H, int I, int bits_gu, int epc, int G,
                             int max_dyn, int* dyn_bytes) {
    const int ck = df_ck(bits_gu), NB = H / 32;
    p = DfPlan{};
    int o = DF_WARPS * DF_NBUF * DF_CODE_SLOT;
    p.sc_slot = df_al(std::max(2 * 16 * (ck / 32) * 2, 16 * (I / 32) * 2), 128);
    p.sc_off = o;
    o += DF_WARPS * DF_NBUF * p.sc_slot;
    p.r1_off = o;
    // phase C
    const int xb = NB * 4 * T * 16;
    p.xc_off = o + xb;
    p.part_off = p.xc_off + NB * 4 * 16;  // C quads [H/32][4]
    p.part_bytes = 2 * 16 * T * 4;
    p.n_part = df_max_tiles(P, E, I, G) + DF_WARPS;
    const int c_end = p.part_off + p.n_part * p.part_bytes;
    // phase D
    p.hs_stride = I * 2 + 16;
    p.hsum_off = o + P * p.hs_stride;
    p.ypair_off = p.hsum_off + P * (I / 32) * 4;
    const int nftr = (H / DF_FT + G - 1) / G;
    const int d_end = p.ypair_off + nftr * P * DF_FT * 4;
    o = df_al(std::max(c_end, d_end), 16);
    p.route_off = o;
    o += df_al((8 * P + 4) * 4, 16);
    p.stab_off = o;  // this layer's row of the slot table
    o += MOE_MAX_E * 4;
    p.bar_off = o;
    o += (DF_WARPS * DF_NBUF + 2) * 8;
    p.total = df_al(o, 128);
    // phase A inside the code ring: x rows [T][2H + 16], W_r rows [epc][4H + 16], sums
    p.a_ws_off = df_al(T * (2 * H + 16), 128);
    p.a_sp_off = df_al(p.a_ws_off + epc * (4 * H + 16), 128);
    p.a_w2_off = p.a_sp_off + DF_WARPS * 64 * 8;
    p.a_xp_off = p.a_w2_off + DF_WARPS * DF_TN * 4;
    // phase B inside the code ring: the records, their keys, the candidate scratch
    // [T][32 ints | 64 doubles] and, for small E, the fallback scratch
    // [T][max(E,32) ints | max(E,64) doubles]
    p.b_rec_off = 0;
    p.b_key_off = T * E * 16;
    p.b_cand_off = p.b_key_off + T * E * 8;
    p.b_fb_stride = df_al(4 * std::max(E, 32), 8) + 8 * std::max(E, 64);
    p.b_fb_off = p.b_fb_stride <= 16 * E ? -1 : p.b_cand_off + T * DF_CAND_BYTES;
    const int b_end = p.b_cand_off + T * DF_CAND_BYTES + (p.b_fb_off < 0 ? 0 : T * p.b_fb_stride);
    *dyn_bytes = 1024 + p.total;
    if (p.a_xp_off + NB * 4 * T * 8 > DF_WARPS * DF_NBUF * DF_CODE_SLOT) return false;
    if (b_end > DF_WARPS * DF_NBUF * DF_CODE_SLOT) return false;
    return *dyn_bytes <= max_dyn;
}

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier over gridDim.x co-resident CTAs, phase `ph` (1, 2, ...):
// thread 0 of every CTA adds one to the counter bar[0] (zeroed before launch,
// it only grows) and polls it until it reaches ph * gridDim.x.  One counter
// costs one atomic round trip plus one polling round trip; 148 arrivals on one
// L2 line serialise in well under that.  Bounded: on expiry the status word
// gets MOE_ERR_TIMEOUT and every thread of the CTA sees false.
// spin_limit bounds the polling (MOE_SPIN_LIMIT unless a test lowers it);
// extra > 0 (a test setting) makes the barrier wait for arrivals that never
// come, so that every waiter runs into that bound.
__device__ __forceinline__ bool grid_barrier(unsigned* bar, unsigned ph, int site, unsigned spin_limit,
                                             unsigned extra = 0) {
    __syncthreads();
    int ok = 1;
    if (threadIdx.x == 0) {
        const unsigned target = ph * (gridDim.x + extra);
        unsigned v;
        // the arrival releases this CTA's writes (ordered before it by the CTA barrier);
        // the last arrival and every waiter acquire everyone else's
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(v) : "l"(bar) : "memory");
        if (v + 1u < target) {
            unsigned it = 0;
            while (ld_acquire_u32(bar) < target) {
                if (++it > spin_limit) { moe_note_timeout(site, (int)(ld_acquire_u32(bar) % 1000)); ok = 0; break; }
            }
        }
    }
    return __syncthreads_and(ok) != 0;
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

// fp16 pairs of 8 codes for the gate/up MMAs.  The exponent-bias pattern
// 0x6400 | v is the fp16 value 1024 + v (ulp 1 at 1024), so a code that sits
// at bit 4 of its field (4-bit: the odd elements; 2-bit: bits 2, 4, 6) gives
// 1024 + m q with m = 16 (or 4, 16, 64) and needs no shift: one LOP3 per
// pair.  The matching x fragment holds x' / m, so each product is
// 1024 x' / m + q x'; the block correction removes the first term and the
// offset.  4-bit: w = codes 0..7 in nibbles, pairs (0,4) m=1, (1,5) m=16,
// (2,6) m=1, (3,7) m=16.  2-bit: bytes `sel` (0x4140: bytes 0-1, 0x4342:
// bytes 2-3) of w hold codes 0..7, pairs (0,4) m=1, (1,5) m=4, (2,6) m=16,
// (3,7) m=64.
template <int BITS>
__device__ __forceinline__ void unpack8_f16(uint32_t w, uint32_t sel, uint32_t (&p)[4]) {
    constexpr uint32_t kMagic = 0x64006400u;
    if (BITS == 4) {
        const uint32_t w8 = w >> 8;
        p[0] = (w & 0x000F000Fu) | kMagic;
        p[1] = (w & 0x00F000F0u) | kMagic;
        p[2] = (w8 & 0x000F000Fu) | kMagic;
        p[3] = (w8 & 0x00F000F0u) | kMagic;
    } else {
        const uint32_t v = __byte_perm(w, 0, sel);  // codes 0-3 in byte 0, codes 4-7 in byte 2
        p[0] = (v & 0x00030003u) | kMagic;
        p[1] = (v & 0x000C000Cu) | kMagic;
        p[2] = (v & 0x00300030u) | kMagic;
        p[3] = (v & 0x00C000C0u) | kMagic;
    }
}

// Factor m of pair i of a gate/up fragment (see unpack8_f16).
template <int BITS>
__host__ __device__ constexpr float df_pair_m(int i) {
    return BITS == 4 ? ((i & 1) ? 16.f : 1.f) : (float)(1 << (2 * i));
}

// D(4 fp32) = A(16x16 f16) * B(16x8 f16) + C (C a separate register quad).
__device__ __forceinline__ void mma_f16_16816_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                uint32_t b0, uint32_t b1, const float4& c) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c.x), "f"(c.y), "f"(c.z), "f"(c.w));
}

// D(4 fp32) += A(16x16 f16) * B(16x8 f16).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(4 fp32) += A(16x16 bf16) * B(16x8 bf16).  (Not volatile: a pure function
// of its operands, which the compiler may schedule freely.)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(4 fp32) = A(16x16 bf16) * B(16x8 bf16) + C, with C a separate register
// quad (loaded as one 16-byte value, so no copies into D are needed).
__device__ __forceinline__ void mma_bf16_16816_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1, const float4& c) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c.x), "f"(c.y), "f"(c.z), "f"(c.w));
}

// Byte offset, inside a 16-row box of 128-byte rows written with the TMA
// 128-byte swizzle, of byte `off` of a row whose swizzle key is
// key16 = (row & 7) << 4: the swizzle XORs the 16-byte chunk index with the
// row's low 3 bits.
__device__ __forceinline__ int sw128(int off, int key16) { return ((off & ~15) ^ key16) | (off & 15); }

// 8 codes of thread q in quant block j of a row: 4 bytes at 4 bits, 2 at 2 bits.
template <int BITS>
__device__ __forceinline__ uint32_t ld_codes(const uint8_t* row, int j, int q, int key16) {
    const int off = j * (32 * BITS / 8) + q * BITS;
    const uint8_t* p = row + (off >> 7) * 2048 + sw128(off & 127, key16);
    if (BITS == 4) return *reinterpret_cast<const uint32_t*>(p);
    return *reinterpret_cast<const uint16_t*>(p);
}

// Four 8x8 b16 matrices from shared memory: lane l gives the address of row
// l % 8 of matrix l / 8 (16 bytes); register k of lane l receives bytes
// 4 (l % 4) .. 4 (l % 4) + 3 of row l / 4 of matrix k.
__device__ __forceinline__ void ldsm_x4(const void* row_addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(row_addr)));
}

// Position of element i (0..I) of a row of h in the fragment order.
__device__ __forceinline__ int frag_pos(int i) {
    const int e32 = i & 31, i8 = e32 & 7;
    return (i & ~31) + (e32 >> 3) * 8 + (i8 & 3) * 2 + (i8 >> 2);
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2,
                                            int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }
__device__ __forceinline__ uint32_t u4_word(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

struct DfRoute {  // grouping of the window's pairs, identical in every CTA; arrays of P
    int32_t* idx;    // expert of pair p = t*k + j
    float* w;
    int32_t* perm;   // position -> pair
    int32_t* inv;    // pair -> position
    int32_t* u_e;    // selected experts, ascending
    int32_t* u_pos;  // first position of each
    int32_t* u_n;    // pairs of each
    int32_t* u_sl;   // arena slot of each, -1 when the slot table has none
    int32_t* n_uniq;
};

// ---------------------------------------------------------------- phase B: top-k of one token

// Order-preserving integer keys of a logit: key32 of its fp32 rounding (for
// the coarse candidate step) and key64 of the fp64 value itself (an exact
// total order, equal values equal keys).  Both are ALU work: on this part a
// chain of fp64 compares and maxima costs several times more latency.
__device__ __forceinline__ uint32_t df_key32(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ unsigned long long df_key64(double d) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(d);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// The single-warp path with its exact fallback, for a token whose candidates do
// not certify: rare, so it is a call rather than inlined code in the kernel.
__device__ __noinline__ void df_topk_fallback(const TopkArgs& a, int t, int32_t* idx_out, float* w_out, int* cs,
                                              double* cvs, int32_t* nrechk) {
    topk_token<2>(a, t, idx_out, w_out, cs, cvs, nrechk);
}

// The selection of topk_token<2> with a shorter first step.  Lanes read the
// (logit, error bound) records of experts e = lane + 32 i from this CTA's
// shared-memory copy.  Every entry whose fp32 key is at or above theta, the
// M-th largest of the 32 lane-maximum keys, is a candidate: at least M entries
// (the lane maxima themselves) reach theta, so the candidates contain the M
// largest in fp32, and every entry left out is below them by the fp32 rounding
// at most - the certification below uses the exact upper end of everything
// left out (rounded up to fp32), so a candidate set that misses a member of the
// true top k only fails it.  With at most 32 candidates they are sorted by
// (exact fp64 value desc, expert asc), one per lane, and certified as in
// topk_token; otherwise, or when the certification fails, topk_token<2>
// decides from scratch (its exact fallback included).
__device__ __forceinline__ void df_topk_token(const TopkArgs& a, const double2* rec, const uint2* reck, int t,
                                              int32_t* idx_out, float* w_out, int* cs, double* cvs, int* fcs,
                                              double* fcvs, int32_t* nrechk) {
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;
    const int M = min(min(E, k + MOE_CAND_EXTRA), 32);
    uint32_t km = 0;  // this lane's largest key (invalid entries: key 0)
#pragma unroll 4
    for (int e = lane; e < E; e += 32) km = max(km, reck[e].x);
    int r = 0;  // rank of this lane's maximum (descending, ties by lane)
#pragma unroll 8
    for (int j = 0; j < 32; ++j) {
        const uint32_t o = __shfl_sync(0xffffffffu, km, j);
        r += (o > km || (o == km && j < lane)) ? 1 : 0;
    }
    const uint32_t thk = __shfl_sync(0xffffffffu, km, __ffs(__ballot_sync(0xffffffffu, r == M - 1)) - 1);
    DF_MARK(20);
    int nc = 0;
    float rest = -INFINITY;  // an upper end of everything that is not a candidate
#pragma unroll 4
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const uint2 q = e < E ? reck[e] : make_uint2(0u, __float_as_uint(-INFINITY));
        const bool in = e < E && q.x >= thk;
        const unsigned bm = __ballot_sync(0xffffffffu, in);
        if (in) {
            const int pos = nc + __popc(bm & ((1u << lane) - 1));
            if (pos < 32) {
                const double2 r2 = rec[e];
                cs[pos] = e;
                cvs[pos] = r2.x;
                cvs[32 + pos] = r2.y;
            }
        } else {
            rest = fmaxf(rest, __uint_as_float(q.y));  // the upper end, rounded up to fp32
        }
        nc += __popc(bm);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rest = fmaxf(rest, __shfl_xor_sync(0xffffffffu, rest, o));
    __syncwarp();
    DF_MARK(21);
    if (nc <= 32) {
        double cval = -INFINITY, cbnd = 0.0;
        int ce = 0x7fffffff;
        if (lane < nc) {
            cval = cvs[lane];
            cbnd = cvs[32 + lane];
            ce = cs[lane];
        }
        // position of this candidate in (value desc, expert asc) order, on exact integer keys
        const unsigned long long ck = lane < nc ? df_key64(cval) : 0ull;
        const uint32_t ckh = (uint32_t)(ck >> 32), ckl = (uint32_t)ck;
        int rank = 0;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
            const uint32_t oh = __shfl_sync(0xffffffffu, ckh, j), ol = __shfl_sync(0xffffffffu, ckl, j);
            const int ej = __shfl_sync(0xffffffffu, ce, j);
            const unsigned long long ok2 = ((unsigned long long)oh << 32) | ol;
            rank += (j < nc && (ok2 > ck || (ok2 == ck && ej < ce))) ? 1 : 0;
        }
        __syncwarp();
        if (lane < nc) {  // scatter into sorted order through the scratch
            cvs[rank] = cval;
            cvs[32 + rank] = cbnd;
            cs[rank] = ce;
        }
        __syncwarp();
        if (lane < nc) {
            cval = cvs[lane];
            cbnd = cvs[32 + lane];
            ce = cs[lane];
        }
        const bool ok = certify_sorted(cval, cbnd, nc, k, (double)rest);
        DF_MARK(22);
        if (ok) {
            write_topk(k, cval, ce, idx_out, w_out);
            return;
        }
    }
    __syncwarp();
    DF_MARK(23);
    df_topk_fallback(a, t, idx_out, w_out, fcs, fcvs, nrechk);
}

// ---------------------------------------------------------------- phase C: one gate/up unit

// A unit is 16 rows x CK = 1024 / BITS codes of W_g and of W_u (one 128-byte
// box row each) and their scales.  Lane (g, q) keeps the codes it feeds to the
// MMA (rows g and g + 8; at 2 bits two blocks share a word) and its scales.
template <int BITS>
struct DfCRegs {
    static constexpr int NB = 32 / BITS;  // quant blocks per unit
    uint32_t g0[8], g1[8], u0[8], u1[8];
    uint4 sg0[NB / 8], sg1[NB / 8], su0[NB / 8], su1[NB / 8];
};

template <int BITS>
__device__ __forceinline__ void df_stage_c(const uint8_t* code, const uint8_t* sc, DfCRegs<BITS>& r) {
    constexpr int NB = DfCRegs<BITS>::NB, NS = NB / 8;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, key16 = (g & 7) << 4;
    if (BITS == 4) {
        // block j of gate rows 0-7 / 8-15, up rows 0-7 / 8-15: one 16-byte chunk per row
        const int rr = lane & 7;
        const uint8_t* rowp = code + (lane >> 4) * 2048 + ((lane >> 3) & 1) * 1024 + rr * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) ldsm_x4(rowp + ((j ^ rr) << 4), r.g0[j], r.g1[j], r.u0[j], r.u1[j]);
    } else {
        const uint8_t* rg0 = code + g * 128;
        const uint8_t* ru0 = code + 2048 + g * 128;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            r.g0[w] = ld_codes<2>(rg0, 2 * w, q, key16) | (ld_codes<2>(rg0, 2 * w + 1, q, key16) << 16);
            r.g1[w] = ld_codes<2>(rg0 + 1024, 2 * w, q, key16) | (ld_codes<2>(rg0 + 1024, 2 * w + 1, q, key16) << 16);
            r.u0[w] = ld_codes<2>(ru0, 2 * w, q, key16) | (ld_codes<2>(ru0, 2 * w + 1, q, key16) << 16);
            r.u1[w] = ld_codes<2>(ru0 + 1024, 2 * w, q, key16) | (ld_codes<2>(ru0 + 1024, 2 * w + 1, q, key16) << 16);
        }
    }
    const uint4* sg = reinterpret_cast<const uint4*>(sc);  // [16 rows][NB] fp16, gate then up
    const uint4* su = sg + 16 * NS;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        r.sg0[i] = sg[g * NS + i];
        r.sg1[i] = sg[(g + 8) * NS + i];
        r.su0[i] = su[g * NS + i];
        r.su1[i] = su[(g + 8) * NS + i];
    }
}

__device__ __forceinline__ float df_scale(const uint4* s, int j) {
    const uint32_t w = u4_word(s[j >> 3], (j & 7) >> 1);
    return (j & 1) ? half_hi(w) : half_lo(w);
}

// accg / accu (rows g, g + 8; token columns 2q, 2q + 1) += the unit's blocks
// J0 .. J0 + NB - 1, in units of the scaled x'.  xb: fp16 x fragments
// [H/32][4][T] (x' / m, see unpack8_f16); xc: per (block, lane q) the MMA's C
// quad (c_2q, c_2q+1, c_2q, c_2q+1), c = -sum over the block of
// (1024 + offset m) x' / m.
template <int BITS>
__device__ __forceinline__ void df_compute_c(const DfCRegs<BITS>& r, const uint4* xb, const float4* xc, int J0, int T,
                                             float (&accg)[4], float (&accu)[4]) {
    constexpr int NB = DfCRegs<BITS>::NB;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        const int J = J0 + j;
        // lanes g >= T load another token's fragment (or, at the last block, the first
        // bytes of xc, which follows xb): it only feeds MMA columns >= T, never stored
        const uint4 bx = xb[(J * 4 + q) * T + g];
        const float4 c = xc[J * 4 + q];
        const uint32_t sel = (j & 1) ? 0x4342u : 0x4140u;  // 2-bit: the block's half of the word
        const int wi = BITS == 2 ? (j >> 1) : j;
        uint32_t pg0[4], pg1[4], pu0[4], pu1[4];
        unpack8_f16<BITS>(r.g0[wi], sel, pg0);
        unpack8_f16<BITS>(r.g1[wi], sel, pg1);
        unpack8_f16<BITS>(r.u0[wi], sel, pu0);
        unpack8_f16<BITS>(r.u1[wi], sel, pu1);
        float dg[4], du[4];
        mma_f16_16816_c(dg, pg0[0], pg1[0], pg0[1], pg1[1], bx.x, bx.y, c);
        mma_f16_16816_c(du, pu0[0], pu1[0], pu0[1], pu1[1], bx.x, bx.y, c);
        mma_f16_16816(dg, pg0[2], pg1[2], pg0[3], pg1[3], bx.z, bx.w);
        mma_f16_16816(du, pu0[2], pu1[2], pu0[3], pu1[3], bx.z, bx.w);
        const float sg0 = df_scale(r.sg0, j), sg1 = df_scale(r.sg1, j);
        const float su0 = df_scale(r.su0, j), su1 = df_scale(r.su1, j);
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

// ---------------------------------------------------------------- phase D: one expert, one feature tile

// acc (features g, g + 8; pair columns 2q, 2q + 1) = W_d rows ft .. ft + 15 x h
// of the expert's n pairs, straight from the slot in a loop of two blocks per
// step, unrolled twice: a W_d unit is used once per launch, so its code stays
// small instead of being unrolled over all blocks.  The unit's codes sit as
// [16 rows][nbox 128-byte chunks] with the TMA 128-byte swizzle keyed on the
// 128-byte line index (row * nbox + chunk); scales as [16 rows][nblk] fp16;
// hs: h of the first pair [n][hstride bytes] in fragment order; hsum: per pair
// and block, the sum of its 32 h values.
template <int BD, int nblk>
__device__ __forceinline__ void df_compute_d_smem(const uint8_t* code, const uint8_t* sc, const uint8_t* hs, int hstride,
                                                  const float* hsum, int n, float (&acc)[4]) {
    constexpr int nbox = nblk * BD / 32;
    constexpr float kOff = 128.f + (float)(1 << (BD - 1));
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, key16 = (g & 7) << 4;
    const bool col_ok = g < n, ok0 = 2 * q < n, ok1 = 2 * q + 1 < n;
    const int mrow = ((lane >> 3) & 1) * 8 + (lane & 7), jo = lane >> 4;  // ldmatrix row address of this lane
    const uint8_t* hrow = hs + g * hstride + q * 16;
#pragma unroll 2
    for (int j = 0; j < nblk; j += 2) {
        uint32_t c[2][2];  // [block j, j + 1][row g, g + 8]
        if (BD == 4) {
            const int jj = j + jo, line = mrow * nbox + (jj >> 3);
            ldsm_x4(code + line * 128 + (((jj & 7) ^ (line & 7)) << 4), c[0][0], c[0][1], c[1][0], c[1][1]);
        } else {
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                c[z][0] = ld_codes<BD>(code + g * 128, j + z, q, key16);
                c[z][1] = ld_codes<BD>(code + g * 128 + 1024, j + z, q, key16);
            }
        }
        const uint32_t sw0 = *reinterpret_cast<const uint32_t*>(sc + (g * nblk + j) * 2);  // rows g, g + 8
        const uint32_t sw1 = *reinterpret_cast<const uint32_t*>(sc + ((g + 8) * nblk + j) * 2);
#pragma unroll
        for (int z = 0; z < 2; ++z) {
            const int jb = j + z;
            uint4 bx = make_uint4(0u, 0u, 0u, 0u);
            if (col_ok) bx = *reinterpret_cast<const uint4*>(hrow + jb * 64);
            const float h0 = ok0 ? hsum[(2 * q) * nblk + jb] : 0.f;
            const float h1 = ok1 ? hsum[(2 * q + 1) * nblk + jb] : 0.f;
            uint32_t p0[4], p1[4];
            unpack8<BD>(c[z][0], p0);
            unpack8<BD>(c[z][1], p1);
            float d[4] = {-kOff * h0, -kOff * h1, -kOff * h0, -kOff * h1};
            mma_bf16_16816(d, p0[0], p1[0], p0[1], p1[1], bx.x, bx.y);
            mma_bf16_16816(d, p0[2], p1[2], p0[3], p1[3], bx.z, bx.w);
            const float s0 = z ? half_hi(sw0) : half_lo(sw0), s1 = z ? half_hi(sw1) : half_lo(sw1);
            acc[0] = fmaf(s0, d[0], acc[0]);
            acc[1] = fmaf(s0, d[1], acc[1]);
            acc[2] = fmaf(s1, d[2], acc[2]);
            acc[3] = fmaf(s1, d[3], acc[3]);
        }
    }
}

// ---------------------------------------------------------------- the kernel

// Device-side pointers into the shared-memory plan, common to both kernels.
struct DfSmem {
    uint8_t* base;
    uint8_t* ring;
    DfRoute rt;
    uint64_t* full;  // [DF_WARPS][DF_NBUF] unit slots
    uint64_t* abar;  // x rows (and the slot-table row); records
    uint64_t* wbar;  // W_r rows
    int32_t* stab;
};

__device__ __forceinline__ DfSmem df_smem(uint8_t* smem_raw, const DfPlan& pl, int P) {
    DfSmem m;
    // 1024-byte aligned base, derived by pointer arithmetic so that every access
    // through it compiles to a shared-memory (not generic) load or store
    m.base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    m.ring = m.base;
    m.rt.idx = reinterpret_cast<int32_t*>(m.base + pl.route_off);
    m.rt.w = reinterpret_cast<float*>(m.rt.idx + P);
    m.rt.perm = reinterpret_cast<int32_t*>(m.rt.w + P);
    m.rt.inv = m.rt.perm + P;
    m.rt.u_e = m.rt.inv + P;
    m.rt.u_pos = m.rt.u_e + P;
    m.rt.u_n = m.rt.u_pos + P;
    m.rt.u_sl = m.rt.u_n + P;
    m.rt.n_uniq = m.rt.u_sl + P;
    m.full = reinterpret_cast<uint64_t*>(m.base + pl.bar_off);
    m.abar = m.full + DF_WARPS * DF_NBUF;
    m.wbar = m.abar + 1;
    m.stab = reinterpret_cast<int32_t*>(m.base + pl.stab_off);
    return m;
}

// ---------------------------------------------------------------- the kernel

template <int BGU, int BD, int NBD>
__global__ void __launch_bounds__(DF_THREADS, 1)
    k_decode_fused(const __grid_constant__ CUtensorMap tgu, const __grid_constant__ CUtensorMap tcd,
                   const __grid_constant__ CUtensorMap tsg, const __grid_constant__ CUtensorMap tsd,
                   DecodeFusedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    constexpr int CK = df_ck(BGU), NBU = CK / 32;  // codes and quant blocks per gate/up unit
    const DfPlan& pl = a.pl;
    const int H = a.H, I = a.I, E = a.E, k = a.k, T = a.T, P = T * k, NB = H / 32;
    DfSmem sm = df_smem(smem_raw, pl, P);
    uint8_t* base = sm.base;
    uint8_t* ring = sm.ring;            // code slots [warp][DF_NBUF][DF_CODE_SLOT]
    uint8_t* scr = base + pl.sc_off;    // scale slots [warp][DF_NBUF][sc_slot]
    uint4* xb = reinterpret_cast<uint4*>(base + pl.r1_off);
    float4* xc = reinterpret_cast<float4*>(base + pl.xc_off);
    float* part = reinterpret_cast<float*>(base + pl.part_off);
    DfRoute& rt = sm.rt;
    uint64_t* full = sm.full;
    uint64_t* abar = sm.abar;
    uint64_t* wbar = sm.wbar;
    const int32_t* stab = sm.stab;
    __shared__ float s_xnorm[DF_TN];
    __shared__ float s_wn[DF_MAX_EPC];
    __shared__ float s_xsc[DF_TN], s_xinv[DF_TN];  // per token: x' = x * s_xsc, a power of two
    __shared__ int s_ustart[DF_WARPS + 1];  // first gate/up unit of each warp
    const int G = gridDim.x, cta = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        tma_prefetch_desc(&tgu);
        tma_prefetch_desc(&tcd);
        tma_prefetch_desc(&tsg);
        tma_prefetch_desc(&tsd);
        for (int i = 0; i < DF_WARPS * DF_NBUF; ++i) mbar_init(&full[i], 1);
        mbar_init(abar, 1);
        mbar_init(wbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    DF_MARK(0);

    // ---- A: router logits in fp64 on the tensor cores.  This CTA takes experts
    // e0 .. e0 + epc - 1 (rows of mma.m8n8k4.f64); its warps split H.  Every
    // bf16 x fp32 product is exact in fp64, so only the additions round
    // (bound: gamma_(H+32)).  The x rows and the W_r rows come in by bulk copies.
    const int epc = a.epc, e0 = cta * epc;
    const int ne = e0 < E ? min(epc, E - e0) : 0;
    const int xstride = 2 * H + 16, wstride = 4 * H + 16;  // padded rows: conflict-free fragment loads
    uint8_t* xs = ring;
    uint8_t* ws = ring + pl.a_ws_off;
    if (tid == 0) {
        // the arrival completes the phase at once when ne == 0 (no bytes expected)
        mbar_arrive_expect_tx(wbar, (uint32_t)(ne * 4 * H));
        for (int e = 0; e < ne; ++e) bulk_load(ws + e * wstride, a.W + (size_t)(e0 + e) * H, (uint32_t)(4 * H), wbar);
        mbar_arrive_expect_tx(abar, (uint32_t)(T * 2 * H + E * 4));
        for (int t = 0; t < T; ++t) bulk_load(xs + t * xstride, a.x + (size_t)t * H, (uint32_t)(2 * H), abar);
        bulk_load(sm.base + pl.stab_off, a.slot_table + (size_t)a.layer * E, (uint32_t)(E * 4), abar);
    }
    bool alive = mbar_wait(abar, 0, 1, 0);
    DF_MARK(1);
    if (warp < T) {  // ||x_t|| for the top-k bounds (inflated over its fp32 rounding), while W_r arrives
        float sq = 0.f;
        for (int i = lane * 8; i < H; i += 256) {
            const uint4 r4 = *reinterpret_cast<const uint4*>(xs + warp * xstride + i * 2);
            const uint32_t wd[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const float lo = __uint_as_float(wd[z] << 16), hi = __uint_as_float(wd[z] & 0xffff0000u);
                sq = fmaf(lo, lo, fmaf(hi, hi, sq));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_xnorm[warp] = sqrtf(sq) * 1.001f;
    }
    // x as fp16 MMA fragments, built while the W_r rows arrive
    {
        const int xstride = 2 * H + 16;
        const uint8_t* xs = ring;
        if (warp < T) {  // per token a power of two that puts max |x| in [2^13, 2^14): the fp16 range holds x'
            float m = 0.f;
            for (int i = lane * 8; i < H; i += 256) {
                const uint4 r4 = *reinterpret_cast<const uint4*>(xs + warp * xstride + i * 2);
                const uint32_t wd[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
                for (int z = 0; z < 4; ++z)
                    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wd[z] << 16)), fabsf(__uint_as_float(wd[z] & 0xffff0000u))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) {
                int ex = 0;
                const bool fin = m > 0.f && m <= 3.0e38f;  // zero or non-finite rows keep scale 1
                if (fin) frexpf(m, &ex);                    // m in [2^(ex-1), 2^ex)
                const int sh = fin ? 14 - ex : 0;
                s_xsc[warp] = ldexpf(1.f, sh);
                s_xinv[warp] = ldexpf(1.f, -sh);
            }
        } else if (warp < DF_TN && lane == 0) {
            s_xsc[warp] = 1.f;
            s_xinv[warp] = 1.f;
        }
        __syncthreads();
        // x as fp16 MMA B fragments [H/32][4][T] (x' / m per pair, see unpack8_f16)
        // and the block-correction parts
        float* xp = reinterpret_cast<float*>(ring + pl.a_xp_off);  // [H/32][4][T]
        const int nxf = NB * 4 * T;
        constexpr float kOffGU = (float)(1 << (BGU - 1));
        for (int u = tid; u < nxf; u += DF_THREADS) {
            const int n = u % T, q = (u / T) % 4, j = u / (4 * T);
            const uint4 r4 = *reinterpret_cast<const uint4*>(xs + n * xstride + (32 * j + 8 * q) * 2);
            float v[8];
            v[0] = __uint_as_float(r4.x << 16); v[1] = __uint_as_float(r4.x & 0xffff0000u);
            v[2] = __uint_as_float(r4.y << 16); v[3] = __uint_as_float(r4.y & 0xffff0000u);
            v[4] = __uint_as_float(r4.z << 16); v[5] = __uint_as_float(r4.z & 0xffff0000u);
            v[6] = __uint_as_float(r4.w << 16); v[7] = __uint_as_float(r4.w & 0xffff0000u);
            const float sc = s_xsc[n];
            uint32_t fr[4];
            float cs = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // pair i = elements (i, i + 4), factor m
                const float im = 1.f / df_pair_m<BGU>(i);  // exact: a power of two
                const __half2 hv = __floats2half2_rn(v[i] * sc * im, v[i + 4] * sc * im);
                fr[i] = *reinterpret_cast<const uint32_t*>(&hv);
                const float2 bb = __half22float2(hv);
                cs += (1024.f + kOffGU * df_pair_m<BGU>(i)) * (bb.x + bb.y);  // exact products, rounded sum
            }
            xb[u] = make_uint4(fr[0], fr[1], fr[2], fr[3]);
            xp[u] = cs;
        }
        __syncthreads();
        for (int u = tid; u < NB * 4; u += DF_THREADS) {  // block corrections as MMA C quads, zero beyond T
            const int q = u % 4, j = u / 4;
            float sx[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                const int n = 2 * q + z;
                sx[z] = 0.f;
                if (n < T) {
                    const float* pp = xp + (size_t)j * 4 * T + n;
                    sx[z] = ((pp[0] + pp[T]) + pp[2 * T]) + pp[3 * T];
                }
            }
            xc[u] = make_float4(-sx[0], -sx[1], -sx[0], -sx[1]);
        }
    }
    alive = mbar_wait(wbar, 0, 1, 1) && alive;
    DF_MARK(2);
    if (ne > 0) {
        const int g = lane >> 2, q = lane & 3;
        const int kw = H / DF_WARPS, kb = warp * kw;
        const bool erow = g < ne, xrow_ok = g < T;
        const uint8_t* wrow = ws + (erow ? g : 0) * wstride;
        const uint8_t* xrow = xs + (xrow_ok ? g : 0) * xstride;
        // two accumulator chains (even and odd 16-element slices) halve the dependent MMA chain
        double c0 = 0.0, c1 = 0.0, d0 = 0.0, d1 = 0.0;
        float w2 = 0.f;
#pragma unroll 2
        for (int k0 = kb; k0 < kb + kw; k0 += 32) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                // step s of this 16-element slice uses k = k1 + 4 q + s (A and B alike)
                const int k1 = k0 + 16 * half;
                const float4 wv = erow ? *reinterpret_cast<const float4*>(wrow + (k1 + 4 * q) * 4) : make_float4(0, 0, 0, 0);
                const uint2 xv = xrow_ok ? *reinterpret_cast<const uint2*>(xrow + (k1 + 4 * q) * 2) : make_uint2(0, 0);
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
        // expert e0 + g, tokens 2q, 2q+1 (this warp's slice of H)
        double* sp = reinterpret_cast<double*>(ring + pl.a_sp_off);
        sp[(warp * 8 + g) * 8 + 2 * q] = c0 + d0;
        sp[(warp * 8 + g) * 8 + 2 * q + 1] = c1 + d1;
        w2 += __shfl_xor_sync(0xffffffffu, w2, 1);
        w2 += __shfl_xor_sync(0xffffffffu, w2, 2);
        float* sw2 = reinterpret_cast<float*>(ring + pl.a_w2_off);
        if (q == 0) sw2[warp * 8 + g] = w2;
    }
    __syncthreads();
    if (warp == 0 && lane < ne) {  // ||W_r[e]|| of this CTA's experts
        const float* sw2 = reinterpret_cast<const float*>(ring + pl.a_w2_off);
        float s2 = 0.f;
        for (int w = 0; w < DF_WARPS; ++w) s2 += sw2[w * 8 + lane];
        s_wn[lane] = sqrtf(s2) * 1.001f;
        a.wnorm[e0 + lane] = s_wn[lane];
    }
    __syncthreads();
    if (tid < 64 && (tid >> 3) < ne && (tid & 7) < T) {  // logits and their error bounds
        const double* sp = reinterpret_cast<const double*>(ring + pl.a_sp_off);
        const int gg = tid >> 3, t = tid & 7, e = e0 + gg;
        double part4[4] = {0.0, 0.0, 0.0, 0.0};  // four short chains: fp64 adds have a long latency here
#pragma unroll
        for (int w = 0; w < DF_WARPS; ++w) part4[w & 3] += sp[(w * 8 + gg) * 8 + t];
        const double sum = (part4[0] + part4[1]) + (part4[2] + part4[3]);
        const double bb = a.b ? (double)a.b[e] : 0.0;
        const double lg = sum + bb;
        a.logit[(size_t)t * E + e] = lg;
        // every sum along a product's path: at most H + 32 roundings in these
        // sums, H + 2 in the definition's own sequential sum
        const double gam = ((double)(H + 32) + (double)(H + 2)) * 1.1102230246251565e-16 * 1.01;
        const double B = ((double)s_xnorm[t] * (double)s_wn[gg] + fabs(bb)) * 1.001;
        const double lv = order_val(lg), bnd = order_bnd(B * gam + 1e-300);
        const double2 r = make_double2(lv, bnd);
        // what the candidate step of the top-k needs, in integer / fp32 form
        const uint2 rk = make_uint2(df_key32((float)lv), __float_as_uint(__double2float_ru(hi_end(lv, bnd))));
#pragma unroll
        for (int c = 0; c < DF_NREP; ++c) {
            a.rec[((size_t)c * T + t) * E + e] = r;
            a.reck[((size_t)c * T + t) * E + e] = rk;
        }
    }
    DF_MARK(3);
    {
        const bool gb = grid_barrier(a.bar, 1u, 1, a.spin_limit, a.bar1_extra);
        alive = __syncthreads_and(alive && gb) != 0;  // uniform across the CTA
    }
    DF_MARK(4);

    // ---- B: certified top-k of every token (the same result in every CTA) and grouping
    if (alive) {
        // this CTA's copy of the records: one bulk copy into the ring, which
        // phase A no longer uses (the grid barrier ended its reads)
        double2* srec = reinterpret_cast<double2*>(ring + pl.b_rec_off);
        uint2* sreck = reinterpret_cast<uint2*>(ring + pl.b_key_off);
        if (tid == 0) {
            fence_proxy_async_global();  // other CTAs wrote the records with plain stores
            fence_proxy_async_smem();    // and this CTA used the ring through the generic proxy
            const uint32_t bytes = (uint32_t)(T * E * 16), kbytes = (uint32_t)(T * E * 8);
            const uint8_t* src = reinterpret_cast<const uint8_t*>(a.rec + (size_t)(cta % DF_NREP) * T * E);
            const uint8_t* ksrc = reinterpret_cast<const uint8_t*>(a.reck + (size_t)(cta % DF_NREP) * T * E);
            mbar_arrive_expect_tx(abar, bytes + kbytes);
            for (uint32_t o = 0; o < bytes; o += 16384)
                bulk_load(reinterpret_cast<uint8_t*>(srec) + o, src + o, min(16384u, bytes - o), abar);
            for (uint32_t o = 0; o < kbytes; o += 16384)
                bulk_load(reinterpret_cast<uint8_t*>(sreck) + o, ksrc + o, min(16384u, kbytes - o), abar);
        }
        alive = mbar_wait(abar, 1, 3, 0);
        DF_MARK(17);
        if (warp < T) {
            TopkArgs ta{};
            ta.x = a.x; ta.W = a.W; ta.b = a.b; ta.logit = a.logit; ta.wnorm = a.wnorm; ta.xnorm = s_xnorm;
            // phase-A sums: at most H + 32 roundings along any product's path
            ta.gfast = (double)(H + 32) * 1.1102230246251565e-16 * 1.01;
            ta.T = T; ta.H = H; ta.E = E; ta.k = k;
            // candidate scratch of this token; the exact fallback reuses the token's own
            // record row (read by the fast step by then) when it holds max(E,32) ints and
            // max(E,64) doubles, else its own region
            int* cs = reinterpret_cast<int*>(ring + pl.b_cand_off + warp * DF_CAND_BYTES);
            double* cvs = reinterpret_cast<double*>(cs + 32);
            int* fcs = pl.b_fb_off < 0 ? reinterpret_cast<int*>(srec + (size_t)warp * E)
                                       : reinterpret_cast<int*>(ring + pl.b_fb_off + warp * pl.b_fb_stride);
            double* fcvs = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(fcs) + df_al(4 * max(E, 32), 8));
            if (alive)
                df_topk_token(ta, srec + (size_t)warp * E, sreck + (size_t)warp * E, warp, rt.idx + warp * k,
                              rt.w + warp * k, cs, cvs, fcs, fcvs, cta == 0 ? a.nrechk : nullptr);
            if (warp == 0) DF_MARK(18);
            __syncwarp();
            if (alive && lane < k) {
                const int e = rt.idx[warp * k + lane];
                if ((unsigned)e >= (unsigned)E) {  // never produced by the top-k; a guard against a library fault
                    rt.idx[warp * k + lane] = 0;
                    moe_set_status(MOE_ERR_RANGE);
                }
            }
        }
        alive = __syncthreads_and(alive) != 0;
        DF_MARK(5);
    }
    if (alive) {
        // grouping: one warp sorts the pairs by (expert, pair id) and lists the
        // experts; in CTA 0 the other warps count the routing outputs directly
        if (warp == 0) {
            int* se = rt.u_n;  // the experts in sorted order (u_n is written after it is read)
            if (P <= 64) {  // keys e * 64 + p, one or two per lane, ranked with shuffles
                const int k0 = lane < P ? rt.idx[lane] * 64 + lane : 0x7fffffff;
                const int k1 = lane + 32 < P ? rt.idx[lane + 32] * 64 + lane + 32 : 0x7fffffff;
                int r0 = 0, r1 = 0;
#pragma unroll 8
                for (int j = 0; j < 32; ++j) {
                    const int o0 = __shfl_sync(0xffffffffu, k0, j), o1 = __shfl_sync(0xffffffffu, k1, j);
                    r0 += (o0 < k0 ? 1 : 0) + (o1 < k0 ? 1 : 0);
                    r1 += (o0 < k1 ? 1 : 0) + (o1 < k1 ? 1 : 0);
                }
                if (lane < P) { rt.perm[r0] = lane; rt.inv[lane] = r0; se[r0] = k0 >> 6; }
                if (lane + 32 < P) { rt.perm[r1] = lane + 32; rt.inv[lane + 32] = r1; se[r1] = k1 >> 6; }
            } else {
                for (int p = lane; p < P; p += 32) {
                    const int e = rt.idx[p];
                    int r = 0;
#pragma unroll 8
                    for (int q2 = 0; q2 < P; ++q2) {
                        const int f = rt.idx[q2];
                        r += (f < e || (f == e && q2 < p)) ? 1 : 0;
                    }
                    rt.perm[r] = p;
                    rt.inv[p] = r;
                    se[r] = e;
                }
            }
            __syncwarp();
            int nu = 0;
            for (int r0 = 0; r0 < P; r0 += 32) {
                const int r = r0 + lane;
                const int e = r < P ? se[r] : -1;
                const bool first = r < P && (r == 0 || se[r - 1] != e);
                const unsigned m = __ballot_sync(0xffffffffu, first);
                if (first) {
                    const int u = nu + __popc(m & ((1u << lane) - 1));
                    const int64_t sl = stab[e];
                    rt.u_e[u] = e;
                    rt.u_pos[u] = r;
                    rt.u_sl[u] = (sl >= 0 && sl < a.n_slots) ? (int32_t)sl : -1;
                    if (cta == 0 && rt.u_sl[u] < 0 && sl != MOE_SLOT_REMOTE) moe_set_status(MOE_ERR_SLOT);
                }
                nu += __popc(m);
            }
            __syncwarp();
            for (int u = lane; u < nu; u += 32) rt.u_n[u] = (u + 1 < nu ? rt.u_pos[u + 1] : P) - rt.u_pos[u];
            if (lane == 0) *rt.n_uniq = nu;
            DF_MARK(19);
        } else if (cta == 0) {
            for (int e = tid - 32; e <= E; e += DF_THREADS - 32) {  // offsets[e] = pairs on experts below e
                int lt = 0, eq = 0;
#pragma unroll 8
                for (int q2 = 0; q2 < P; ++q2) {
                    const int f = rt.idx[q2];
                    lt += f < e ? 1 : 0;
                    eq += f == e ? 1 : 0;
                }
                a.offsets[e] = lt;
                if (e < E && a.hist) a.hist[(size_t)a.layer * E + e] += (uint32_t)eq;
            }
        }
        __syncthreads();
        if (cta == 0)
            for (int p = tid; p < P; p += DF_THREADS) {
                a.perm[p] = rt.perm[p];
                a.idx[p] = rt.idx[p];
                a.w[p] = rt.w[p];
            }
    }
    DF_MARK(6);
    DF_CLK(cb0);

    // ---- C: gate/up + SwiGLU.  A grid barrier separates C from D, so each phase
    // is balanced on its own: every CTA takes an equal share of the 16-row
    // gate/up tiles, contiguous in (expert, row) order.
    const int tiles_e = I / 16, NCH = H / CK, NFT = H / DF_FT;
    constexpr int nblk_d = NBD, nbox_d = NBD * BD / 32;  // W_d row: quant blocks, 128-byte chunks
    const int nuq = alive ? *rt.n_uniq : 0;
    const int R = nuq * tiles_e;
    const int r0 = (int)((int64_t)cta * R / G), r1 = (int)((int64_t)(cta + 1) * R / G);
    const int nloc = r1 - r0;
    if (nloc + DF_WARPS > pl.n_part) {  // the host's bound on partial slots was wrong
        moe_set_status(MOE_ERR_RANGE);
        alive = false;
    }
    // this warp's units: gate/up units [ub, ue) of the CTA's tiles (tile-major),
    // then W_d units (feature round rr, expert warp + 16 i)
    const int Uc = alive ? nloc * NCH : 0;
    if (tid <= DF_WARPS) s_ustart[tid] = tid * Uc / DF_WARPS;
    const int ub = warp * Uc / DF_WARPS, ue = (warp + 1) * Uc / DF_WARPS;
    const int nC = ue - ub;
    const int nftc = df_nft(cta, NFT, G);
    const int ndw = (alive && nuq > warp) ? (nuq - warp + DF_WARPS - 1) / DF_WARPS : 0;
    const int S = nC + nftc * ndw;
    const uint32_t bytes_c = 2u * 2048u, bytes_d = (uint32_t)(nbox_d * 2048);
    const uint32_t bytes_sc = 2u * 16u * NBU * 2u, bytes_sd = 16u * nblk_d * 2u;  // their scales

    // Units of this warp in order: gate/up units ub .. ue - 1 (unit u = chunk u % NCH
    // of local tile u / NCH; tile r0 + lt is rows r16 * 16 .. +15 of distinct expert
    // ui), then W_d units (feature round rr, expert warp + 16 dd).  The issuing lane
    // and the consuming warp walk them with their own cursors, without divisions.
    struct Cur {
        int lt, ch, ui, r16, rr, dd;
    };
    auto cur_init = [&](Cur& c) {
        const int u = ub, lt = u / max(NCH, 1), gt = r0 + lt;
        c.lt = lt;
        c.ch = u - lt * NCH;
        c.ui = gt / tiles_e;
        c.r16 = gt - c.ui * tiles_e;
        c.rr = 0;
        c.dd = 0;
    };
    auto cur_next = [&](Cur& c, int s_done) {  // s_done: the unit just passed
        if (s_done < nC) {
            if (++c.ch == NCH) {
                c.ch = 0;
                ++c.lt;
                if (++c.r16 == tiles_e) {
                    c.r16 = 0;
                    ++c.ui;
                }
            }
        } else if (++c.dd == ndw) {
            c.dd = 0;
            ++c.rr;
        }
    };

    // Issue unit s (at the issuing cursor) into this warp's slot s % DF_NBUF: one
    // lane starts the TMA loads of its codes and its scales; the slot's barrier
    // completes when both have landed.
    auto issue = [&](int s, const Cur& c) {
        const int b = s % DF_NBUF;
        uint64_t* fb = &full[warp * DF_NBUF + b];
        uint8_t* cdst = ring + (warp * DF_NBUF + b) * DF_CODE_SLOT;
        uint8_t* sdst = scr + (warp * DF_NBUF + b) * pl.sc_slot;
        if (s < nC) {
            const int sl = rt.u_sl[c.ui];
            if (sl < 0) {
                mbar_arrive(fb);  // nothing to load: the unit counts 0
            } else {
                mbar_arrive_expect_tx(fb, bytes_c + bytes_sc);
                tma_load_5d(cdst, &tgu, fb, 0, c.ch, c.r16 * 16, 0, sl);  // gate and up, 16 rows x 128 B each
                tma_load_4d(sdst, &tsg, fb, c.ch * NBU, c.r16 * 16, 0, sl);  // [gate, up][16 rows][NBU] fp16
            }
        } else {
            const int ui = warp + DF_WARPS * c.dd, ft = (cta + c.rr * G) * DF_FT;
            const int sl = rt.u_sl[ui];
            if (sl < 0) {
                mbar_arrive(fb);
            } else {
                mbar_arrive_expect_tx(fb, bytes_d + bytes_sd);
                tma_load_4d(cdst, &tcd, fb, 0, 0, ft, sl);  // 16 rows x nbox_d x 128 B
                tma_load_3d(sdst, &tsd, fb, 0, ft, sl);     // [16 rows][nblk_d] fp16
            }
        }
    };

    int issued = 0;  // units issued by this warp (the same count in every lane)
    Cur ic;          // the issuing lane's cursor
    cur_init(ic);
    if (S > 0) {
        if (lane == 0) {
            fence_proxy_async_smem();  // the ring held generic-proxy data during A and B
            for (int i = 0; i < min(S, DF_NBUF); ++i) {
                issue(i, ic);
                cur_next(ic, i);
            }
        }
        issued = min(S, DF_NBUF);
    }
    DF_CLK(cl0);
    if (nC > 0) DF_WACC(9, cl0 - cb0);
    bool wok = true;
    int s = 0;  // units consumed
    Cur cc;     // the consuming cursor (every lane)
    cur_init(cc);
    {
        float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
        const int g = lane >> 2, q = lane & 3;
        for (; s < nC; ++s) {
            const int b = s % DF_NBUF;
            DF_CLK(c0);
            if (!mbar_wait(&full[warp * DF_NBUF + b], (uint32_t)(s / DF_NBUF) & 1u, 4, s)) { wok = false; break; }
            DF_CLK(c1);
            DF_WACC(0, c1 - c0);
            DF_WACC(4, 1);
            if (s == 0) DF_MARK(10);
            const bool valid = rt.u_sl[cc.ui] >= 0;
            DfCRegs<BGU> cr;
            if (valid)
                df_stage_c<BGU>(ring + (warp * DF_NBUF + b) * DF_CODE_SLOT, scr + (warp * DF_NBUF + b) * pl.sc_slot,
                                cr);
            __syncwarp();  // every lane's reads of the slot are done: it may be refilled
            DF_CLK(c1a);
            DF_WACC(8, c1a - c1);
            if (issued < S) {  // re-arm the slot with unit s + DF_NBUF
                if (lane == 0) {
                    issue(issued, ic);
                    cur_next(ic, issued);
                }
                ++issued;
            }
            DF_CLK(c1b);
            DF_WACC(7, c1b - c1a);
            if (valid) df_compute_c<BGU>(cr, xb, xc, cc.ch * NBU, T, accg, accu);
            DF_CLK(c2);
            DF_WACC(1, c2 - c1);
            if (s == 0) DF_WACC(6, c2 - c1);
            if (s == nC - 1 || cc.ch == NCH - 1) {  // this warp's part of tile lt is complete
                float* pp = part + (size_t)(cc.lt + warp) * (2 * 16 * T);  // [gate, up][16 rows][T]
#pragma unroll
                for (int z = 0; z < 2; ++z) {
                    const int col = 2 * q + z;
                    if (col < T) {  // back from x' to x: an exact power-of-two scaling
                        const float iv = s_xinv[col];
                        pp[g * T + col] = accg[z] * iv;
                        pp[(g + 8) * T + col] = accg[2 + z] * iv;
                        pp[16 * T + g * T + col] = accu[z] * iv;
                        pp[16 * T + (g + 8) * T + col] = accu[2 + z] * iv;
                    }
                }
#pragma unroll
                for (int z = 0; z < 4; ++z) accg[z] = accu[z] = 0.f;
            }
            cur_next(cc, s);
        }
    }
    const bool cok = __syncthreads_and(wok && alive) != 0;
    DF_MARK(11);
    // finish the tiles: sum the partials of the warps that covered each tile (in
    // warp order), SwiGLU, round h to bf16 and store it for every pair of the expert
    if (cok) {
        for (int item = tid; item < nloc * 16 * DF_TN; item += DF_THREADS) {
            const int lt = item / (16 * DF_TN), row = (item / DF_TN) % 16, jj = item % DF_TN;
            const int gt = r0 + lt, ui = gt / tiles_e, r16 = gt % tiles_e;
            if (jj >= rt.u_n[ui]) continue;
            const int pos = rt.u_pos[ui] + jj, t = rt.perm[pos] / k;
            const int u_first = lt * NCH, u_end = u_first + NCH;
            float gs = 0.f, us = 0.f;
            for (int w = 0; w < DF_WARPS; ++w) {  // warps whose units meet the tile, in order
                const int wb = s_ustart[w], we = s_ustart[w + 1];
                if (wb >= we || we <= u_first || wb >= u_end) continue;
                const float* pp = part + (size_t)(lt + w) * (2 * 16 * T);
                gs += pp[row * T + t];
                us += pp[16 * T + row * T + t];
            }
            const float h = silu_f32(gs) * us;
            a.hB[(size_t)pos * I + frag_pos(r16 * 16 + row)] = f32_to_bf16_bits(h);
        }
    }
    DF_MARK(12);
    {
        const bool gb = grid_barrier(a.bar, 2u, 2, a.spin_limit);
        alive = __syncthreads_and(cok && gb) != 0;
    }
    DF_MARK(13);

    // ---- D: down projection of this CTA's feature tiles for every selected
    // expert (warp w takes experts w, w + 16, ...), then the combine.
    uint8_t* hs = base + pl.r1_off;  // h of every pair [P][hs_stride], fragment order
    float* hsum = reinterpret_cast<float*>(base + pl.hsum_off);    // [P][I/32]
    float* ypair = reinterpret_cast<float*>(base + pl.ypair_off);  // [round][P][DF_FT]
    if (alive) {  // h of every pair into shared memory, and per (pair, block) the sum of its 32 h
        for (int it = tid; it < P * nblk_d; it += DF_THREADS) {
            const int p = it / nblk_d, j = it % nblk_d;
            const uint4* src = reinterpret_cast<const uint4*>(a.hB + (size_t)p * I + j * 32);
            uint4 v[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) v[z] = __ldcg(src + z);  // written by other CTAs: read at L2
            uint4* dst = reinterpret_cast<uint4*>(hs + (size_t)p * pl.hs_stride + j * 64);
            float sum = 0.f;
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                dst[z] = v[z];
                const uint32_t wd[4] = {v[z].x, v[z].y, v[z].z, v[z].w};
#pragma unroll
                for (int y = 0; y < 4; ++y) sum += __uint_as_float(wd[y] << 16) + __uint_as_float(wd[y] & 0xffff0000u);
            }
            hsum[it] = sum;
        }
        __syncthreads();
        DF_MARK(14);
    }
    if (alive) {
        const int g = lane >> 2, q = lane & 3;
        for (; s < S; ++s) {
            const int b = s % DF_NBUF;
            DF_CLK(c0);
            if (!mbar_wait(&full[warp * DF_NBUF + b], (uint32_t)(s / DF_NBUF) & 1u, 6, s)) { wok = false; break; }
            DF_CLK(c1);
            DF_WACC(2, c1 - c0);
            DF_WACC(5, 1);
            const int rr = cc.rr, ui = warp + DF_WARPS * cc.dd;
            const int pos0 = rt.u_pos[ui], n = rt.u_n[ui];
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (rt.u_sl[ui] >= 0)
                df_compute_d_smem<BD, NBD>(ring + (warp * DF_NBUF + b) * DF_CODE_SLOT,
                                           scr + (warp * DF_NBUF + b) * pl.sc_slot, hs + (size_t)pos0 * pl.hs_stride,
                                           pl.hs_stride, hsum + (size_t)pos0 * nblk_d, n, acc);
            __syncwarp();  // the slot's reads are done: it may be refilled
            if (issued < S) {
                if (lane == 0) {
                    issue(issued, ic);
                    cur_next(ic, issued);
                }
                ++issued;
            }
            DF_CLK(c2);
            DF_WACC(3, c2 - c1);
#pragma unroll
            for (int z = 0; z < 2; ++z) {  // y for pair columns 2q, 2q+1 (when they exist), features g, g+8
                const int jj = 2 * q + z;
                if (jj < n) {
                    const int pos = pos0 + jj;
                    const float wv = rt.w[rt.perm[pos]];
                    float* yp = ypair + ((size_t)rr * P + pos) * DF_FT;
                    yp[g] = wv * acc[z];
                    yp[g + 8] = wv * acc[2 + z];
                }
            }
            cur_next(cc, s);
        }
        alive = __syncthreads_and(wok) != 0;
        DF_MARK(15);
        if (alive)
            for (int u = tid; u < nftc * T * DF_FT; u += DF_THREADS) {
                const int rr = u / (T * DF_FT), t = (u / DF_FT) % T, fl = u % DF_FT;
                const int f = (cta + rr * G) * DF_FT + fl;
                float sum = 0.f;
                for (int j = 0; j < k; ++j) sum += ypair[((size_t)rr * P + rt.inv[t * k + j]) * DF_FT + fl];
                if (a.residual) sum = bf16_bits_to_f32(a.x[(size_t)t * H + f]) + sum;
                if (a.hout) a.hout[(size_t)t * H + f] = sum;
                else a.out[(size_t)t * H + f] = f32_to_bf16_bits(sum);
            }
    }
    // On an error path, wait (bounded) for this warp's copies still in flight
    // before the CTA's shared memory goes away.
    for (int r = s; r < issued; ++r) mbar_wait(&full[warp * DF_NBUF + r % DF_NBUF], (uint32_t)(r / DF_NBUF) & 1u, 8, r);
    DF_MARK(16);
}
