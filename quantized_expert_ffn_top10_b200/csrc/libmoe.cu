// libmoe.so: the C ABI declared in include/moe.h.  Host code validates every
// argument before the first CUDA call, lays out the caller's workspace, encodes
// TMA descriptors and enqueues the kernels of router.cuh, perm.cuh, decode.cuh
// and prefill.cuh on the caller's stream.  Nothing here allocates memory.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "decode.cuh"
#include "decode_fused.cuh"
#include "perm.cuh"
#include "prefill.cuh"
#include "router.cuh"
#include "router_f64.cuh"
#include "router_tc.cuh"

namespace {

constexpr size_t kAlign = 256;
inline size_t al(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Ws {
    size_t idx, w, logit, absum, cmax, offsets, perm, inv, uniq, meta, chunk, tiles, nrechk, xp, h, y, rec, gbar, wsplit,
        xn, slow, slowrec, last, hout, reck, total;
};

inline int max_tiles(int P, int E) { return (P + PREFILL_TILE_N - 1) / PREFILL_TILE_N + std::min(E, P); }

Ws ws_layout(int T, int E, int k, int H, int I) {
    const size_t P = (size_t)T * k;
    const size_t nch = (P + PERM_CHUNK - 1) / PERM_CHUNK;
    const bool small = T <= MOE_DECODE_MAX_T;
    const bool f64r = T <= MOE_ROUTER_F64_MAX_T;  // fp64 router logits (decode windows and short chunks)
    Ws w{};
    size_t o = 0;
    auto put = [&](size_t bytes) { size_t r = o; o += al(std::max<size_t>(bytes, 1)); return r; };
    w.idx = put(P * 4);
    w.w = put(P * 4);
    w.logit = put((size_t)T * E * (f64r ? 8 : 4));  // fp64 logits up to MOE_ROUTER_F64_MAX_T, fp32 above
    w.absum = put(small ? (size_t)T * E * 8 : 0);
    w.cmax = put((size_t)E * 4);                    // router row norms
    w.offsets = put((size_t)(E + 1) * 4);
    w.perm = put(P * 4);
    w.inv = put(P * 4);
    w.uniq = put((size_t)E * 4);
    w.meta = put(16);
    w.chunk = put(nch * E * 4);
    w.tiles = put((size_t)max_tiles((int)P, E) * 16);
    w.nrechk = put(4);
    w.gbar = put(small ? DF_BAR_WORDS * 4 : 0);  // fused decode: grid barrier (right after nrechk: one memset clears both)
    w.xp = put(P * H * 2);
    w.h = put(P * I * (small ? 4 : 2));  // decode keeps h and Y in fp32, prefill in bf16
    w.y = put(P * H * (small ? 4 : 2));
    w.rec = put(small ? (size_t)DF_NREP * T * E * 16 : 0);  // fused decode: replicated (logit, bound) records
    w.reck = put(small ? (size_t)DF_NREP * T * E * 8 : 0);  // and their keys
    w.wsplit = put(small ? 0 : (size_t)3 * E * H * 2);        // chunk router: W_r as three bf16 planes
    w.xn = put(small ? 0 : (size_t)T * 4);                     // chunk router: ||x_t|| per token
    w.slow = put(small ? 0 : (size_t)(T + 4) * 4);             // chunk top-k: [count, tokens...] left to the slow pass
    w.slowrec = put(small ? 0 : (size_t)T * sizeof(SlowRec));  // and the fast pass's candidates of each
    w.last = put(small ? 0 : (size_t)(T + 4) * 4);             // [count, tokens...] left to the last pass
    w.hout = put(small ? (size_t)T * H * 4 : 0);               // fused decode + steering: fp32 output rows
    w.total = o;
    return w;
}

// ---------------------------------------------------------------- process state

std::mutex g_mu;
std::vector<cudaEvent_t> g_stage_ev;  // measurement hook, see moe_set_stage_events
std::atomic<uint64_t> g_launches{0};
uint64_t g_init_mask[4] = {0, 0, 0, 0};  // devices whose kernel attributes are set
int g_df_grid[256];                     // fused-decode grid (one CTA per SM) per device, 0 = unusable
int g_df_maxdyn[256];                   // its dynamic shared-memory limit per device
std::atomic<unsigned> g_dbg_spin{0};    // test setting: grid-barrier polling bound (0 = MOE_SPIN_LIMIT)
std::atomic<unsigned> g_dbg_bar1{0};    // test setting: extra arrivals grid barrier 1 waits for
constexpr int kDfMaxH = 2560;           // largest H the fused decode kernel stages

inline void stage(int i, cudaStream_t st) {
    std::lock_guard<std::mutex> g(g_mu);
    if ((int)g_stage_ev.size() <= i) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(g_stage_ev[i], st, cudaEventRecordExternal);  // an event-record node of the graph
    else
        cudaEventRecord(g_stage_ev[i], st);
}

inline void count(int n) { g_launches += (uint64_t)n; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_desc(const moe_arena_desc* d, bool prefill) {
    if (!d) return MOE_ERR_ARG;
    if (d->block != 32 || d->reserved != 0) return MOE_ERR_SHAPE;
    if (d->H < 32 || d->H > 8192 || d->H % 32 || d->I < 32 || d->I > 4096 || d->I % 32) return MOE_ERR_SHAPE;
    if (prefill && (d->H % 128 || d->I % 128)) return MOE_ERR_SHAPE;
    const int bits[3] = {d->bits_gate, d->bits_up, d->bits_down};
    if (d->slot_bytes <= 0 || d->slot_bytes % 256 || d->n_slots < 1) return MOE_ERR_SHAPE;
    for (int m = 0; m < 3; ++m) {
        if (bits[m] != 2 && bits[m] != 4) return MOE_ERR_SHAPE;
        const int64_t rows = m < 2 ? d->I : d->H, K = m < 2 ? d->H : d->I;
        const int64_t cb = rows * K * bits[m] / 8, sb = rows * (K / 32) * 2;
        if (d->off_codes[m] < 0 || d->off_codes[m] % 128 || d->off_codes[m] + cb > d->slot_bytes) return MOE_ERR_SHAPE;
        if (d->off_scales[m] < 0 || d->off_scales[m] % 128 || d->off_scales[m] + sb > d->slot_bytes)
            return MOE_ERR_SHAPE;
    }
    return MOE_OK;
}

int check_route_args(const uint16_t* x, int T, int H, const float* W, int E, int k, const void* ws, int maxT) {
    if (T < 0 || T > maxT) return MOE_ERR_RANGE;
    if (E < 1 || E > MOE_MAX_E || k < 1 || k > std::min(E, MOE_MAX_TOPK)) return MOE_ERR_RANGE;
    if (H < 32 || H > 8192 || H % 32) return MOE_ERR_SHAPE;
    if (!x || !W || !ws) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(W, 16) || !aligned(ws, kAlign)) return MOE_ERR_ARG;
    return MOE_OK;
}

// gamma_n = n u / (1 - n u): bound factor of a sum whose terms pass through at most n roundings
inline double gamma_n(int n, double u) { return (double)n * u / (1.0 - (double)n * u); }

inline int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

bool tmap_bf16_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int box_rows);
bool g_router_tc_ok[256];  // the tensor-core router kernel may run on this device (set by ensure_init)

// Router + grouping on the caller's stream.  idx/w/offsets/perm may be the
// caller's buffers or workspace.
int launch_route(const uint16_t* x, int T, int H, const float* W, const float* b, int E, int k, int32_t* idx,
                 float* w, int32_t* offsets, int32_t* perm, int32_t* nrechk, uint8_t* ws, const Ws& L, bool want_tiles,
                 uint32_t* hist, int layer, cudaStream_t st) {
    const int P = T * k;
    int32_t* nr = nrechk ? nrechk : reinterpret_cast<int32_t*>(ws + L.nrechk);
    if (cudaMemsetAsync(nr, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    TopkArgs ta{};
    ta.x = x; ta.W = W; ta.b = b; ta.logit = ws + L.logit; ta.idx = idx; ta.w = w; ta.n_rechecked = nr;
    ta.T = T; ta.H = H; ta.E = E; ta.k = k;
    const int tk_grid = (T + MOE_TOPK_WARPS - 1) / MOE_TOPK_WARPS;
    if (T <= MOE_DECODE_MAX_T) {
        double* logit = reinterpret_cast<double*>(ws + L.logit);
        double* absum = reinterpret_cast<double*>(ws + L.absum);
        k_router_gemv<<<(E + 7) / 8, 256, 0, st>>>(x, T, H, W, b, E, logit, absum);
        ta.absum = absum;
        ta.gfast = gamma_n(H / 32 + 6, 1.1102230246251565e-16);
        k_topk<1><<<tk_grid, 32 * MOE_TOPK_WARPS, 0, st>>>(ta);
    } else if (T <= MOE_ROUTER_F64_MAX_T) {  // short chunk: fp64 tensor-core logits, bound from norms
        double* logit = reinterpret_cast<double*>(ws + L.logit);
        float* wnorm = reinterpret_cast<float*>(ws + L.cmax);
        k_router_f64<<<dim3((E + 7) / 8, (T + 7) / 8), 32 * RF_WARPS, 0, st>>>(x, T, H, W, b, E, logit, wnorm);
        ta.wnorm = wnorm;
        ta.gfast = (double)(H + 32) * 1.1102230246251565e-16 * 1.01;
        k_topk<2><<<tk_grid, 32 * MOE_TOPK_WARPS, 0, st>>>(ta);
    } else {
        float* wnorm = reinterpret_cast<float*>(ws + L.cmax);
        float* logit = reinterpret_cast<float*>(ws + L.logit);
        int dev = 0;
        cudaGetDevice(&dev);
        CUtensorMap tmA, tmB;
        uint16_t* planes = reinterpret_cast<uint16_t*>(ws + L.wsplit);
        const bool tc = dev >= 0 && dev < 256 && g_router_tc_ok[dev] && E % RT_BM == 0 && H % RT_BK == 0 &&
                        L.wsplit + (size_t)3 * E * H * 2 <= L.total && tmap_bf16_rows(&tmA, planes, 3LL * E, H, RT_BM) &&
                        tmap_bf16_rows(&tmB, x, T, H, RT_BN);
        if (tc) {  // tensor cores: W_r as three exact bf16 planes, fp32 accumulation in TMEM
            k_router_split<<<E, 256, 0, st>>>(W, E, H, planes, wnorm);
            k_router_tc<<<dim3(E / RT_BM, (T + RT_BN - 1) / RT_BN), RT_THREADS, RT_SMEM, st>>>(tmA, tmB, T, H, E, b,
                                                                                              logit);
            ta.gfast = moe_tc_router_gamma(H);
        } else {
            k_router_norms<<<(E + 7) / 8, 256, 0, st>>>(W, E, H, wnorm);
            k_router_gemm<<<dim3((E + RG_BN - 1) / RG_BN, (T + RG_BM - 1) / RG_BM), 256, 0, st>>>(x, T, H, W, b, E,
                                                                                                  logit);
            ta.gfast = gamma_n(RG_BK + H / RG_BK + 2, 5.9604644775390625e-8);
        }
        ta.wnorm = wnorm;
        float* xn = reinterpret_cast<float*>(ws + L.xn);
        k_xnorm<<<(T + 7) / 8, 256, 0, st>>>(x, T, H, xn);
        ta.xnorm = xn;
        ta.slow_count = reinterpret_cast<int32_t*>(ws + L.slow);
        ta.slow_list = ta.slow_count + 4;
        ta.slow_rec = reinterpret_cast<SlowRec*>(ws + L.slowrec);
        ta.last_count = reinterpret_cast<int32_t*>(ws + L.last);
        ta.last_list = ta.last_count + 4;
        if (cudaMemsetAsync(ta.slow_count, 0, 4, st) != cudaSuccess ||
            cudaMemsetAsync(ta.last_count, 0, 4, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        k_topk_fast<0><<<tk_grid, 32 * MOE_TOPK_WARPS, 0, st>>>(ta);
        k_topk_slow<<<std::min(T, 4 * 148), 32 * MOE_SLOW_WARPS, 0, st>>>(ta);
        k_topk_last<<<tk_grid, 32 * MOE_TOPK_WARPS, 0, st>>>(ta);
    }
    PermArgs pa{};
    pa.idx = idx; pa.P = P; pa.E = E; pa.nchunks = (P + PERM_CHUNK - 1) / PERM_CHUNK;
    pa.chunk_cnt = reinterpret_cast<int32_t*>(ws + L.chunk);
    pa.offsets = offsets; pa.perm = perm;
    pa.inv = reinterpret_cast<int32_t*>(ws + L.inv);
    pa.uniq = reinterpret_cast<int32_t*>(ws + L.uniq);
    pa.meta = reinterpret_cast<int32_t*>(ws + L.meta);
    pa.tiles = want_tiles ? reinterpret_cast<int4*>(ws + L.tiles) : nullptr;
    pa.hist = hist; pa.layer = layer;
    k_perm_count<<<pa.nchunks, PERM_CHUNK, 0, st>>>(pa);
    k_perm_scan<<<1, MOE_MAX_E, 0, st>>>(pa);
    k_perm_scatter<<<pa.nchunks, PERM_CHUNK, 0, st>>>(pa);
    count(T <= MOE_ROUTER_F64_MAX_T ? 5 : 9);
    return cuda_rc(cudaGetLastError());
}

// ---------------------------------------------------------------- TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

// bf16 [rows][K] row-major, box 64 x box_rows, 128-byte swizzle; rows past the end read as zero
bool tmap_bf16_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int box_rows) {
    if (!encoder()) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Gate and up codes of every slot as one 5-D tensor: (128-byte chunk, chunk
// index, row, matrix, slot); a box is 16 rows x one chunk of both matrices,
// landing as [matrix][row][128 B] with the 128-byte swizzle.
bool tmap_codes_gu(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t row_bytes, int64_t mat_stride,
                   int64_t n_slots, int64_t slot_bytes) {
    cuuint64_t dims[5] = {128, (cuuint64_t)(row_bytes / 128), (cuuint64_t)rows, 2, (cuuint64_t)n_slots};
    cuuint64_t strides[4] = {128, (cuuint64_t)row_bytes, (cuuint64_t)mat_stride, (cuuint64_t)slot_bytes};
    cuuint32_t box[5] = {128, 1, 16, 2, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<uint8_t*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W_d codes of every slot as a 4-D tensor (128-byte chunk, chunk index, row,
// slot); a box is 16 rows x all chunks of a row, landing as [row][chunk][128 B].
bool tmap_codes_d(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t row_bytes, int64_t n_slots,
                  int64_t slot_bytes) {
    cuuint64_t dims[4] = {128, (cuuint64_t)(row_bytes / 128), (cuuint64_t)rows, (cuuint64_t)n_slots};
    cuuint64_t strides[3] = {128, (cuuint64_t)row_bytes, (cuuint64_t)slot_bytes};
    cuuint32_t box[4] = {128, (cuuint32_t)(row_bytes / 128), 16, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Gate and up scales of every slot as one 4-D fp16 tensor (block, row, matrix,
// slot); a box is nblk blocks of 16 rows of both matrices, landing as
// [matrix][row][nblk].
bool tmap_scales_gu(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t nblk_row, int64_t mat_stride,
                    int64_t n_slots, int64_t slot_bytes, int nblk) {
    cuuint64_t dims[4] = {(cuuint64_t)nblk_row, (cuuint64_t)rows, 2, (cuuint64_t)n_slots};
    cuuint64_t strides[3] = {(cuuint64_t)nblk_row * 2, (cuuint64_t)mat_stride, (cuuint64_t)slot_bytes};
    cuuint32_t box[4] = {(cuuint32_t)nblk, 16, 2, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<uint8_t*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W_d scales of every slot as a 3-D fp16 tensor (block, row, slot); a box is
// the whole scale row of 16 rows, landing as [row][nblk].
bool tmap_scales_d(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t nblk_row, int64_t n_slots,
                   int64_t slot_bytes) {
    cuuint64_t dims[3] = {(cuuint64_t)nblk_row, (cuuint64_t)rows, (cuuint64_t)n_slots};
    cuuint64_t strides[2] = {(cuuint64_t)nblk_row * 2, (cuuint64_t)slot_bytes};
    cuuint32_t box[3] = {(cuuint32_t)nblk_row, 16, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<uint8_t*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// ---------------------------------------------------------------- process state

// Raise the dynamic shared-memory limit of every large-smem kernel, once per
// device, so that later calls (and graph captures) only launch.
int ensure_init() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_mu);
    if (g_init_mask[dev >> 6] >> (dev & 63) & 1ull) return MOE_OK;
    const int dsm = MOE_DECODE_MAX_T * 8192 * 2, dnm = MOE_DECODE_MAX_T * 4096 * 4;
    cudaError_t e = cudaSuccess;
    auto chk = [&](cudaError_t r) { if (r != cudaSuccess) e = r; };
    chk(set_smem(k_dec_gateup<4, 4>, dsm)); chk(set_smem(k_dec_gateup<2, 2>, dsm));
    chk(set_smem(k_dec_gateup<2, 4>, dsm)); chk(set_smem(k_dec_gateup<4, 2>, dsm));
    chk(set_smem(k_dec_down<4>, dnm)); chk(set_smem(k_dec_down<2>, dnm));
    chk(set_smem(k_prefill_gemm<0, 4, 4>, PfCfg<0>::SMEM)); chk(set_smem(k_prefill_gemm<0, 2, 2>, PfCfg<0>::SMEM));
    chk(set_smem(k_prefill_gemm<0, 2, 4>, PfCfg<0>::SMEM)); chk(set_smem(k_prefill_gemm<0, 4, 2>, PfCfg<0>::SMEM));
    chk(set_smem(k_prefill_gemm<1, 4, 4>, PfCfg<1>::SMEM)); chk(set_smem(k_prefill_gemm<1, 2, 2>, PfCfg<1>::SMEM));
    // fused decode: all the shared memory a CTA can have, less the kernel's static arrays
    cudaFuncAttributes fa{};
    chk(cudaFuncGetAttributes(&fa, k_decode_fused<4, 4, 16>));
    const int dfs = DF_SMEM_LIMIT - (int)fa.sharedSizeBytes;
    chk(set_smem(k_decode_fused<4, 4, 16>, dfs)); chk(set_smem(k_decode_fused<4, 4, 8>, dfs));
    chk(set_smem(k_decode_fused<4, 2, 16>, dfs)); chk(set_smem(k_decode_fused<2, 4, 16>, dfs));
    chk(set_smem(k_decode_fused<2, 4, 8>, dfs)); chk(set_smem(k_decode_fused<2, 2, 16>, dfs));
    int nsm = 0, per = 0;
    chk(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    chk(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k_decode_fused<4, 4, 16>, DF_THREADS, dfs));
    g_df_grid[dev] = (per >= 1) ? nsm : 0;
    g_df_maxdyn[dev] = dfs;
    g_router_tc_ok[dev] = set_smem(k_router_tc, RT_SMEM) == cudaSuccess;
    if (e != cudaSuccess || !encoder()) return MOE_ERR_CUDA;
    g_init_mask[dev >> 6] |= 1ull << (dev & 63);
    return MOE_OK;
}

}  // namespace

// ---------------------------------------------------------------- decode / prefill drivers

namespace {

struct LayerCall {
    const moe_arena_desc* d;
    const uint8_t* arena;
    const int32_t* slot_table;
    int L, layer;
    const uint16_t* x;
    int T;
    const float* W;
    const float* b;
    int E, k, residual;
    const float* steer;
    uint16_t* out;
    uint32_t* hist;
    const moe_route_out* ro;
    uint8_t* ws;
    size_t ws_bytes;
    cudaStream_t st;
    float* part;  // expert parallelism: fp32 partial sums instead of out (no residual, no steering)
};

int check_layer(const LayerCall& c, bool prefill) {
    int rc = check_desc(c.d, prefill);
    if (rc) return rc;
    rc = check_route_args(c.x, c.T, c.d->H, c.W, c.E, c.k, c.ws, prefill ? MOE_PREFILL_MAX_T : MOE_DECODE_MAX_T);
    if (rc) return rc;
    if (c.L < 1 || c.layer < 0 || c.layer >= c.L) return MOE_ERR_RANGE;
    if (!c.arena || !c.slot_table || (!c.out && !c.part)) return MOE_ERR_ARG;
    if (!aligned(c.arena, 256) || !aligned(c.out, 16) || !aligned(c.steer, 16) || !aligned(c.part, 16))
        return MOE_ERR_ARG;
    if (c.out) {
        const size_t xb = (size_t)c.T * c.d->H * 2;
        const uintptr_t x0 = reinterpret_cast<uintptr_t>(c.x), o0 = reinterpret_cast<uintptr_t>(c.out);
        if (c.T > 0 && x0 < o0 + xb && o0 < x0 + xb) return MOE_ERR_ARG;
    }
    if (c.ws_bytes < ws_layout(c.T, c.E, c.k, c.d->H, c.d->I).total) return MOE_ERR_WS;
    return MOE_OK;
}

struct Routed {
    int32_t *idx, *offsets, *perm;
    float* w;
};

int route_for_layer(const LayerCall& c, const Ws& L, bool tiles, Routed& r) {
    const moe_route_out* ro = c.ro;
    r.idx = (ro && ro->topk_idx) ? ro->topk_idx : reinterpret_cast<int32_t*>(c.ws + L.idx);
    r.w = (ro && ro->topk_w) ? ro->topk_w : reinterpret_cast<float*>(c.ws + L.w);
    r.offsets = (ro && ro->expert_offsets) ? ro->expert_offsets : reinterpret_cast<int32_t*>(c.ws + L.offsets);
    r.perm = (ro && ro->perm) ? ro->perm : reinterpret_cast<int32_t*>(c.ws + L.perm);
    return launch_route(c.x, c.T, c.d->H, c.W, c.b, c.E, c.k, r.idx, r.w, r.offsets, r.perm,
                        ro ? ro->n_rechecked : nullptr, c.ws, L, tiles, c.hist, c.layer, c.st);
}

template <int BG, int BU>
void launch_gateup(const DecodeArgs& a, int umax, int T, cudaStream_t st) {
    const int smem = T * a.H * 2;
    k_dec_gateup<BG, BU><<<dim3((a.I + 31) / 32, umax), 32 * DEC_GU_WARPS, smem, st>>>(a);
}

template <int BD>
void launch_down(const DecodeArgs& a, int umax, int T, cudaStream_t st) {
    const int smem = T * a.I * 4;
    k_dec_down<BD><<<dim3((a.H + 31) / 32, umax), 32 * DEC_DN_WARPS, smem, st>>>(a);
}

// Shapes the fused decode kernel stages: gate/up K-chunks of min(H, 1024)
// with 128-byte code rows per chunk and 16-byte scale rows; down rows of
// 128-byte multiples; everything within one ring slot and the smem plan.
// Whether the fused decode kernel takes this window; fills its shared-memory plan.
bool fused_decode_ok(const moe_arena_desc* d, int T, int E, int k, DfPlan* plan, int* dyn, int* epc) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || g_df_grid[dev] < 1) return false;
    const int H = d->H, I = d->I, G = g_df_grid[dev];
    if (d->bits_gate != d->bits_up) return false;  // one unit shape for gate and up
    if (d->off_codes[1] <= d->off_codes[0]) return false;  // gate and up codes as one tensor
    if (d->off_scales[1] <= d->off_scales[0] || (d->off_scales[1] - d->off_scales[0]) % 16 ||
        d->off_scales[0] % 16 || d->off_scales[2] % 16)
        return false;  // gate and up scales as one tensor; every scale tensor 16-byte aligned
    if (T > DF_TN || T * k > DF_MAXP || E > MOE_MAX_E || H > kDfMaxH) return false;
    if (H % df_ck(d->bits_gate) || H % 256 || I % 256 || I / 32 > DF_MAX_NBD) return false;
    const int wd_row = I * d->bits_down / 8;  // bytes of a W_d row: one or two 128-byte boxes
    if (wd_row % 128 || wd_row > DF_CODE_SLOT / 16) return false;
    if (E % 4) return false;  // the slot-table row arrives by one bulk copy (16-byte multiple)
    *epc = (E + G - 1) / G;
    if (*epc > DF_MAX_EPC) return false;
    return df_plan(*plan, T, T * k, E, H, I, d->bits_gate, *epc, G, g_df_maxdyn[dev], dyn);
}

template <int BGU, int BD, int NBD>
cudaError_t launch_fused(const CUtensorMap* tm, const DecodeFusedArgs& a, int grid, int dyn, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DF_THREADS);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;  // all CTAs co-resident: the grid barriers rely on it
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_decode_fused<BGU, BD, NBD>, tm[0], tm[1], tm[2], tm[3], a);
}

int run_decode_fused(const LayerCall& c, const DfPlan& plan, int dyn, int epc) {
    const moe_arena_desc* d = c.d;
    const int H = d->H, I = d->I;
    const Ws L = ws_layout(c.T, c.E, c.k, H, I);
    const moe_route_out* ro = c.ro;
    int dev = 0;
    cudaGetDevice(&dev);
    DecodeFusedArgs a{};
    a.arena = c.arena; a.slot_table = c.slot_table; a.n_slots = d->n_slots; a.slot_bytes = d->slot_bytes;
    for (int m = 0; m < 3; ++m) { a.off_codes[m] = d->off_codes[m]; a.off_scales[m] = d->off_scales[m]; }
    a.H = H; a.I = I; a.E = c.E; a.k = c.k; a.layer = c.layer; a.T = c.T; a.residual = c.part ? 0 : c.residual;
    a.bits_gate = d->bits_gate; a.bits_up = d->bits_up; a.bits_down = d->bits_down;
    a.epc = epc;
    a.x = c.x; a.W = c.W; a.b = c.b; a.out = c.out; a.hist = c.hist;
    a.hout = c.part ? c.part : c.steer ? reinterpret_cast<float*>(c.ws + L.hout) : nullptr;
    a.idx = (ro && ro->topk_idx) ? ro->topk_idx : reinterpret_cast<int32_t*>(c.ws + L.idx);
    a.w = (ro && ro->topk_w) ? ro->topk_w : reinterpret_cast<float*>(c.ws + L.w);
    a.offsets = (ro && ro->expert_offsets) ? ro->expert_offsets : reinterpret_cast<int32_t*>(c.ws + L.offsets);
    a.perm = (ro && ro->perm) ? ro->perm : reinterpret_cast<int32_t*>(c.ws + L.perm);
    a.nrechk = (ro && ro->n_rechecked) ? ro->n_rechecked : reinterpret_cast<int32_t*>(c.ws + L.nrechk);
    a.logit = reinterpret_cast<double*>(c.ws + L.logit);
    a.wnorm = reinterpret_cast<float*>(c.ws + L.cmax);
    a.hB = reinterpret_cast<uint16_t*>(c.ws + L.h);
    a.bar = reinterpret_cast<unsigned int*>(c.ws + L.gbar);
    a.rec = reinterpret_cast<double2*>(c.ws + L.rec);
    a.reck = reinterpret_cast<uint2*>(c.ws + L.reck);
    a.pl = plan;
    a.spin_limit = g_dbg_spin.load() ? g_dbg_spin.load() : MOE_SPIN_LIMIT;
    a.bar1_extra = g_dbg_bar1.load();
    CUtensorMap tm[4];
    const int64_t ns = d->n_slots, sb = d->slot_bytes;
    if (!tmap_codes_gu(&tm[0], c.arena + d->off_codes[0], I, (int64_t)H * d->bits_gate / 8,
                       d->off_codes[1] - d->off_codes[0], ns, sb) ||
        !tmap_codes_d(&tm[1], c.arena + d->off_codes[2], H, (int64_t)I * d->bits_down / 8, ns, sb) ||
        !tmap_scales_gu(&tm[2], c.arena + d->off_scales[0], I, H / 32, d->off_scales[1] - d->off_scales[0], ns, sb,
                        df_ck(d->bits_gate) / 32) ||
        !tmap_scales_d(&tm[3], c.arena + d->off_scales[2], H, I / 32, ns, sb))
        return MOE_ERR_CUDA;
    // the grid barrier's words and the recheck counter start at zero: one memset when the
    // counter is the workspace's own (it sits just before the barrier words), else two
    int32_t* const ws_nr = reinterpret_cast<int32_t*>(c.ws + L.nrechk);
    if (a.nrechk == ws_nr) {
        if (cudaMemsetAsync(ws_nr, 0, (L.gbar - L.nrechk) + DF_BAR_WORDS * 4, c.st) != cudaSuccess) return MOE_ERR_CUDA;
    } else if (cudaMemsetAsync(a.bar, 0, DF_BAR_WORDS * 4, c.st) != cudaSuccess ||
               cudaMemsetAsync(a.nrechk, 0, 4, c.st) != cudaSuccess) {
        return MOE_ERR_CUDA;
    }
    stage(0, c.st);
    const int grid = g_df_grid[dev];
    cudaError_t e;
    switch (d->bits_gate * 1000 + d->bits_down * 100 + I / 32) {  // I / 32 blocks per W_d row
        case 4416: e = launch_fused<4, 4, 16>(tm, a, grid, dyn, c.st); break;
        case 4408: e = launch_fused<4, 4, 8>(tm, a, grid, dyn, c.st); break;
        case 4216: e = launch_fused<4, 2, 16>(tm, a, grid, dyn, c.st); break;
        case 2416: e = launch_fused<2, 4, 16>(tm, a, grid, dyn, c.st); break;
        case 2408: e = launch_fused<2, 4, 8>(tm, a, grid, dyn, c.st); break;
        default: e = launch_fused<2, 2, 16>(tm, a, grid, dyn, c.st); break;
    }
    if (e == cudaSuccess && c.steer && !c.part) {  // steering: the rows leave the kernel in fp32, one block per token finishes them
        k_combine_steer<float><<<c.T, STEER_THREADS, H * 4, c.st>>>(nullptr, nullptr, nullptr, a.hout, c.T, H, c.k, 0,
                                                                    c.steer, c.out);
        count(1);
    }
    stage(1, c.st);  // one kernel: only its start and end are recorded
    count(1);
    return e == cudaSuccess ? cuda_rc(cudaGetLastError()) : MOE_ERR_CUDA;
}

int run_decode(const LayerCall& c) {
    DfPlan plan;
    int dyn = 0, epc = 0;
    if (aligned(c.slot_table, 16) && fused_decode_ok(c.d, c.T, c.E, c.k, &plan, &dyn, &epc))
        return run_decode_fused(c, plan, dyn, epc);
    const moe_arena_desc* d = c.d;
    const Ws L = ws_layout(c.T, c.E, c.k, d->H, d->I);
    Routed r;
    stage(0, c.st);
    int rc = route_for_layer(c, L, false, r);
    if (rc) return rc;
    stage(1, c.st);
    DecodeArgs a{};
    a.arena = c.arena; a.slot_table = c.slot_table; a.slot_bytes = d->slot_bytes; a.n_slots = d->n_slots;
    for (int m = 0; m < 3; ++m) { a.off_codes[m] = d->off_codes[m]; a.off_scales[m] = d->off_scales[m]; }
    a.H = d->H; a.I = d->I; a.E = c.E; a.k = c.k; a.layer = c.layer;
    a.x = c.x; a.offsets = r.offsets; a.perm = r.perm;
    a.uniq = reinterpret_cast<int32_t*>(c.ws + L.uniq);
    a.meta = reinterpret_cast<int32_t*>(c.ws + L.meta);
    a.topk_w = r.w;
    a.h = reinterpret_cast<float*>(c.ws + L.h);
    a.y = reinterpret_cast<float*>(c.ws + L.y);
    const int umax = std::min(c.E, c.T * c.k);
    if (d->bits_gate == 4 && d->bits_up == 4) launch_gateup<4, 4>(a, umax, c.T, c.st);
    else if (d->bits_gate == 2 && d->bits_up == 2) launch_gateup<2, 2>(a, umax, c.T, c.st);
    else if (d->bits_gate == 2) launch_gateup<2, 4>(a, umax, c.T, c.st);
    else launch_gateup<4, 2>(a, umax, c.T, c.st);
    stage(2, c.st);
    if (d->bits_down == 4) launch_down<4>(a, umax, c.T, c.st);
    else launch_down<2>(a, umax, c.T, c.st);
    stage(3, c.st);
    if (c.part)
        k_combine_f32<float><<<dim3((d->H / 4 + 127) / 128, c.T), 128, 0, c.st>>>(
            a.y, reinterpret_cast<int32_t*>(c.ws + L.inv), c.T, d->H, c.k, c.part);
    else if (c.steer)
        k_combine_steer<float><<<c.T, STEER_THREADS, d->H * 4, c.st>>>(
            c.x, a.y, reinterpret_cast<int32_t*>(c.ws + L.inv), nullptr, c.T, d->H, c.k, c.residual, c.steer, c.out);
    else
        k_combine<float><<<dim3((d->H / 4 + 127) / 128, c.T), 128, 0, c.st>>>(
            c.x, a.y, reinterpret_cast<int32_t*>(c.ws + L.inv), c.T, d->H, c.k, c.residual, c.out);
    stage(4, c.st);
    count(3);
    return cuda_rc(cudaGetLastError());
}

// The activation matrix [rows][K] bf16 seen through boxes of 128, 64, 32 and 16 rows.
struct ActMaps {
    CUtensorMap m[4];
    bool make(const void* base, int64_t rows, int64_t K) {
        return tmap_bf16_rows(&m[0], base, rows, K, 128) && tmap_bf16_rows(&m[1], base, rows, K, 64) &&
               tmap_bf16_rows(&m[2], base, rows, K, 32) && tmap_bf16_rows(&m[3], base, rows, K, 16);
    }
};

// mgroups CTAs per N-tile, each over mtiles / mgroups M-tiles (mgroups divides mtiles).
template <int MODE, int B0, int B1>
void launch_gemm(const ActMaps& t, PrefillArgs a, int mtiles, int mgroups, int ntile_max, cudaStream_t st) {
    while (mtiles % mgroups) --mgroups;
    a.mgroups = mgroups;
    k_prefill_gemm<MODE, B0, B1><<<ntile_max * mgroups, PF_THREADS, PfCfg<MODE>::SMEM, st>>>(t.m[0], t.m[1], t.m[2],
                                                                                             t.m[3], a);
}

int run_prefill(const LayerCall& c) {
    const moe_arena_desc* d = c.d;
    const int H = d->H, I = d->I, P = c.T * c.k;
    const Ws L = ws_layout(c.T, c.E, c.k, H, I);
    if (!encoder()) return MOE_ERR_CUDA;
    Routed r;
    stage(0, c.st);
    int rc = route_for_layer(c, L, true, r);
    if (rc) return rc;
    stage(1, c.st);
    uint16_t* xp = reinterpret_cast<uint16_t*>(c.ws + L.xp);
    uint16_t* h = reinterpret_cast<uint16_t*>(c.ws + L.h);
    uint16_t* y = reinterpret_cast<uint16_t*>(c.ws + L.y);
    k_gather_rows<<<(P + GATHER_ROWS - 1) / GATHER_ROWS, 32 * GATHER_ROWS, 0, c.st>>>(c.x, r.perm, P, H, c.k, xp);
    ActMaps tx, th;
    const int64_t ns = d->n_slots, sb = d->slot_bytes;
    if (!tx.make(xp, P, H) || !th.make(h, P, I)) return MOE_ERR_CUDA;
    PrefillArgs a{};
    a.arena = c.arena; a.slot_table = c.slot_table; a.n_slots = ns; a.slot_bytes = sb;
    for (int m = 0; m < 3; ++m) { a.off_codes[m] = d->off_codes[m]; a.off_scales[m] = d->off_scales[m]; }
    a.H = H; a.I = I; a.E = c.E; a.k = c.k; a.layer = c.layer;
    a.tiles = reinterpret_cast<const int4*>(c.ws + L.tiles);
    a.meta = reinterpret_cast<const int32_t*>(c.ws + L.meta);
    a.perm = r.perm; a.topk_w = r.w;
    const int nt = max_tiles(P, c.E);
    a.out = h;
    // CTAs per N-tile: GEMM1 one per M-tile (the CTAs of a tile are adjacent, so they read its
    // activation rows together and share them through L2), GEMM2 one per 8 M-tiles (measured
    // best at H = 2048, I = 512)
    const int mg1 = std::max(1, I / PF_BM), mg2 = std::max(1, H / PF_BM / 8);
    if (d->bits_gate == 4 && d->bits_up == 4) launch_gemm<0, 4, 4>(tx, a, I / PF_BM, mg1, nt, c.st);
    else if (d->bits_gate == 2 && d->bits_up == 2) launch_gemm<0, 2, 2>(tx, a, I / PF_BM, mg1, nt, c.st);
    else if (d->bits_gate == 2) launch_gemm<0, 2, 4>(tx, a, I / PF_BM, mg1, nt, c.st);
    else launch_gemm<0, 4, 2>(tx, a, I / PF_BM, mg1, nt, c.st);
    stage(2, c.st);
    a.out = y;
    if (d->bits_down == 4) launch_gemm<1, 4, 4>(th, a, H / PF_BM, mg2, nt, c.st);
    else launch_gemm<1, 2, 2>(th, a, H / PF_BM, mg2, nt, c.st);
    stage(3, c.st);
    if (c.part)
        k_combine_f32<uint16_t><<<dim3((H / 4 + 127) / 128, c.T), 128, 0, c.st>>>(
            y, reinterpret_cast<int32_t*>(c.ws + L.inv), c.T, H, c.k, c.part);
    else if (c.steer)
        k_combine_steer<uint16_t><<<c.T, STEER_THREADS, H * 4, c.st>>>(
            c.x, y, reinterpret_cast<int32_t*>(c.ws + L.inv), nullptr, c.T, H, c.k, c.residual, c.steer, c.out);
    else
        k_combine_bf16x8<<<dim3((H / 8 + 127) / 128, c.T), 128, 0, c.st>>>(
            c.x, y, reinterpret_cast<int32_t*>(c.ws + L.inv), c.T, H, c.k, c.residual, c.out);
    stage(4, c.st);
    count(4);
    return cuda_rc(cudaGetLastError());
}

}  // namespace

// ---------------------------------------------------------------- exported entry points

extern "C" {

size_t moe_workspace_bytes(int T, int E, int top_k, int H, int I) {
    if (T < 0 || E < 1 || top_k < 1 || H < 1 || I < 1) return 0;
    // the layout grows with T inside each router regime; across a regime's upper
    // limit it can shrink, so the size is the largest over every T' <= T
    size_t b = ws_layout(T, E, top_k, H, I).total;
    for (const int lim : {MOE_DECODE_MAX_T, MOE_ROUTER_F64_MAX_T})
        if (T > lim) b = std::max(b, ws_layout(lim, E, top_k, H, I).total);
    return b;
}

int moe_route(const uint16_t* x, int T, int H, const float* router_w, const float* router_bias, int E, int top_k,
              int32_t* topk_idx, float* topk_w, int32_t* expert_offsets, int32_t* perm, void* ws, size_t ws_bytes,
              void* stream) {
    int rc = check_route_args(x, T, H, router_w, E, top_k, ws, MOE_PREFILL_MAX_T);
    if (rc) return rc;
    if (!topk_idx || !topk_w || !expert_offsets || !perm) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    const Ws L = ws_layout(T, E, top_k, H, 32);
    if (ws_bytes < L.total) return MOE_ERR_WS;
    if (T > MOE_DECODE_MAX_T && (rc = ensure_init()) != MOE_OK) return rc;  // the chunk router's kernel attributes
    return launch_route(x, T, H, router_w, router_bias, E, top_k, topk_idx, topk_w, expert_offsets, perm, nullptr,
                        static_cast<uint8_t*>(ws), L, false, nullptr, 0, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// Scratch of moe_route_static: one fixed array per device, no allocation.
static __device__ __align__(256) uint8_t g_route_scratch[MOE_ROUTE_STATIC_BYTES];

namespace {
// Per device: the address of g_route_scratch and the CUDA context it was
// looked up in.  A different current context on the device (after
// cudaDeviceReset, or a context the caller made current) has its own copy of
// the array, so the address is looked up again there.
void* g_route_scratch_addr[256];
CUcontext g_route_scratch_ctx[256];

PFN_cuCtxGetCurrent_v4000 ctx_getter() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    });
    return fn;
}

// Address of g_route_scratch in the current context of the current device.
// The first call in a context does the lookup (cudaGetSymbolAddress); later
// calls in that context only compare the context handle.
int route_scratch(uint8_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return MOE_ERR_CUDA;
    CUcontext ctx = nullptr;
    PFN_cuCtxGetCurrent_v4000 get = ctx_getter();
    if (!get || get(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_mu);
    if (!ctx || !g_route_scratch_addr[dev] || g_route_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        // (also makes the device's primary context current when no context is)
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        if (!aligned(p, kAlign)) return MOE_ERR_CUDA;
        if (get(&ctx) != CUDA_SUCCESS || !ctx) return MOE_ERR_CUDA;
        g_route_scratch_addr[dev] = p;
        g_route_scratch_ctx[dev] = ctx;
    }
    *out = static_cast<uint8_t*>(g_route_scratch_addr[dev]);
    return MOE_OK;
}
}  // namespace

extern "C" {

int moe_route_static(const uint16_t* x, int T, int H, const float* router_w, const float* router_bias, int E,
                     int top_k, int32_t* topk_idx, float* topk_w, int32_t* expert_offsets, int32_t* perm,
                     void* stream) {
    if (T > MOE_ROUTE_STATIC_MAX_T) return MOE_ERR_STATIC;
    int rc = check_route_args(x, T, H, router_w, E, top_k, reinterpret_cast<const void*>(kAlign),
                              MOE_ROUTE_STATIC_MAX_T);
    if (rc) return rc;
    if (!topk_idx || !topk_w || !expert_offsets || !perm) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    const Ws L = ws_layout(T, E, top_k, H, 32);
    if (L.xp > MOE_ROUTE_STATIC_BYTES) return MOE_ERR_STATIC;  // the router and grouping use [0, xp) only
    uint8_t* scratch = nullptr;
    rc = route_scratch(&scratch);
    if (rc) return rc;
    return launch_route(x, T, H, router_w, router_bias, E, top_k, topk_idx, topk_w, expert_offsets, perm, nullptr,
                        scratch, L, false, nullptr, 0, static_cast<cudaStream_t>(stream));
}

static int forward(bool prefill, const moe_arena_desc* desc, const void* arena, const int32_t* slot_table, int L,
                   int layer, const uint16_t* x, int T, const float* router_w, const float* router_bias, int E,
                   int top_k, int residual, const float* steer, uint16_t* out, uint32_t* hist,
                   const moe_route_out* route_out, void* ws, size_t ws_bytes, void* stream, float* part = nullptr) {
    LayerCall c{desc, static_cast<const uint8_t*>(arena), slot_table, L, layer, x, T, router_w, router_bias, E,
                top_k, residual, steer, out, hist, route_out, static_cast<uint8_t*>(ws), ws_bytes,
                static_cast<cudaStream_t>(stream), part};
    int rc = check_layer(c, prefill);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    rc = ensure_init();
    if (rc) return rc;
    return prefill ? run_prefill(c) : run_decode(c);
}

int moe_forward_decode(const moe_arena_desc* desc, const void* arena, const int32_t* slot_table, int L, int layer,
                       const uint16_t* x, int T, const float* router_w, const float* router_bias, int E, int top_k,
                       int residual, const float* steer, uint16_t* out, uint32_t* hist, const moe_route_out* route_out,
                       void* ws, size_t ws_bytes, void* stream) {
    return forward(false, desc, arena, slot_table, L, layer, x, T, router_w, router_bias, E, top_k, residual, steer, out,
                   hist, route_out, ws, ws_bytes, stream);
}

int moe_forward_prefill(const moe_arena_desc* desc, const void* arena, const int32_t* slot_table, int L, int layer,
                        const uint16_t* x, int T, const float* router_w, const float* router_bias, int E, int top_k,
                        int residual, const float* steer, uint16_t* out, uint32_t* hist, const moe_route_out* route_out,
                        void* ws, size_t ws_bytes, void* stream) {
    return forward(true, desc, arena, slot_table, L, layer, x, T, router_w, router_bias, E, top_k, residual, steer, out,
                   hist, route_out, ws, ws_bytes, stream);
}

int moe_forward_partial(int prefill, const moe_arena_desc* desc, const void* arena, const int32_t* slot_table, int L,
                        int layer, const uint16_t* x, int T, const float* router_w, const float* router_bias, int E,
                        int top_k, float* partial, uint32_t* hist, const moe_route_out* route_out, void* ws,
                        size_t ws_bytes, void* stream) {
    if (!partial) return MOE_ERR_ARG;
    return forward(prefill != 0, desc, arena, slot_table, L, layer, x, T, router_w, router_bias, E, top_k, 0, nullptr,
                   nullptr, hist, route_out, ws, ws_bytes, stream, partial);
}

int moe_finish_rows(const uint16_t* x, const float* sum, int T, int H, int residual, const float* steer, uint16_t* out,
                    void* stream) {
    if (!sum || !out || (residual && !x)) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(sum, 16) || !aligned(steer, 16) || !aligned(out, 16)) return MOE_ERR_ARG;
    if (T < 0 || H < 8 || H > 8192 || H % 8) return MOE_ERR_SHAPE;
    if (T == 0) return MOE_OK;
    const int rc = ensure_init();
    if (rc) return rc;
    k_finish_rows<<<T, STEER_THREADS, H * 4, static_cast<cudaStream_t>(stream)>>>(x, sum, T, H, residual, steer, out);
    count(1);
    return cuda_rc(cudaGetLastError());
}

int moe_route_histogram(const int32_t* expert_offsets, int E, int L, int layer, uint32_t* hist, void* stream) {
    if (!expert_offsets || !hist) return MOE_ERR_ARG;
    if (E < 1 || E > MOE_MAX_E || L < 1 || layer < 0 || layer >= L) return MOE_ERR_RANGE;
    k_hist_add<<<(E + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(expert_offsets, E, layer, hist);
    count(1);
    return cuda_rc(cudaGetLastError());
}

int moe_rank_experts(const uint32_t* hist_host, int L, int E, uint16_t* pairs_out) {
    if (!hist_host || !pairs_out) return MOE_ERR_ARG;
    if (L < 1 || E < 1 || E > MOE_MAX_E || L > 65535) return MOE_ERR_RANGE;
    const int n = L * E;
    std::vector<int32_t> order(n);
    for (int i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(),
                     [&](int32_t a, int32_t b) { return hist_host[a] > hist_host[b]; });
    for (int r = 0; r < n; ++r) {
        pairs_out[2 * r] = (uint16_t)(order[r] / E);
        pairs_out[2 * r + 1] = (uint16_t)(order[r] % E);
    }
    return MOE_OK;
}

// ---------------------------------------------------------------- expert profile (STRP v1)

int64_t moe_profile_bytes(int n_pairs, int L, int E) {
    if (L < 1 || E < 1 || L > 65535 || E > 65535 || n_pairs < 0 || (int64_t)n_pairs > (int64_t)L * E) return -1;
    return 4 + 5 * 4 + (int64_t)n_pairs * 4 + (int64_t)L * E * 4;
}

namespace {
inline void put_u32(uint8_t* p, uint32_t v) { for (int i = 0; i < 4; ++i) p[i] = (uint8_t)(v >> (8 * i)); }
inline void put_u16(uint8_t* p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
inline uint32_t get_u32(const uint8_t* p) { return p[0] | (p[1] << 8) | (p[2] << 16) | ((uint32_t)p[3] << 24); }
inline uint16_t get_u16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
}  // namespace

int64_t moe_profile_write(const uint16_t* pairs, int n_pairs, int L, int E, uint8_t* buf, size_t buf_bytes) {
    const int64_t need = moe_profile_bytes(n_pairs, L, E);
    if (need < 0) return MOE_ERR_RANGE;
    if (!buf) return need;
    if (!pairs && n_pairs > 0) return MOE_ERR_ARG;
    if (buf_bytes < (size_t)need) return MOE_ERR_WS;
    std::vector<int32_t> inv((size_t)L * E, -1);
    for (int r = 0; r < n_pairs; ++r) {
        const int l = pairs[2 * r], e = pairs[2 * r + 1];
        if (l >= L || e >= E || inv[(size_t)l * E + e] >= 0) return MOE_ERR_ARG;  // out of range or ranked twice
        inv[(size_t)l * E + e] = r;
    }
    uint8_t* p = buf;
    p[0] = 'S'; p[1] = 'T'; p[2] = 'R'; p[3] = 'P';
    put_u32(p + 4, 1);                          // version
    put_u32(p + 8, (uint32_t)L);                // layers
    put_u32(p + 12, (uint32_t)E);               // experts per layer
    put_u32(p + 16, (uint32_t)n_pairs);         // ranked pairs
    put_u32(p + 20, (uint32_t)((int64_t)L * E));  // entries of the inverse tables
    p += 24;
    for (int r = 0; r < n_pairs; ++r, p += 4) {
        put_u16(p, pairs[2 * r]);
        put_u16(p + 2, pairs[2 * r + 1]);
    }
    for (size_t i = 0; i < inv.size(); ++i, p += 4) put_u32(p, (uint32_t)inv[i]);
    return need;
}

int moe_profile_read(const uint8_t* buf, size_t bytes, int* L, int* E, int* n_pairs, uint16_t* pairs,
                     int32_t* inverse) {
    if (!buf || !L || !E || !n_pairs) return MOE_ERR_ARG;
    if (bytes < 24 || buf[0] != 'S' || buf[1] != 'T' || buf[2] != 'R' || buf[3] != 'P') return MOE_ERR_SHAPE;
    if (get_u32(buf + 4) != 1) return MOE_ERR_SHAPE;
    const uint32_t l = get_u32(buf + 8), e = get_u32(buf + 12), n = get_u32(buf + 16), ent = get_u32(buf + 20);
    if (l < 1 || e < 1 || l > 65535 || e > 65535 || (uint64_t)n > (uint64_t)l * e || (uint64_t)ent != (uint64_t)l * e)
        return MOE_ERR_SHAPE;
    if ((int64_t)bytes != moe_profile_bytes((int)n, (int)l, (int)e)) return MOE_ERR_SHAPE;
    *L = (int)l; *E = (int)e; *n_pairs = (int)n;
    const uint8_t* p = buf + 24;
    for (uint32_t r = 0; r < n; ++r, p += 4) {
        const uint16_t pl = get_u16(p), pe = get_u16(p + 2);
        if (pl >= l || pe >= e) return MOE_ERR_SHAPE;
        if (pairs) { pairs[2 * r] = pl; pairs[2 * r + 1] = pe; }
    }
    for (uint64_t i = 0; i < ent; ++i, p += 4) {
        const int32_t v = (int32_t)get_u32(p);
        if (v < -1 || v >= (int32_t)n) return MOE_ERR_SHAPE;
        if (inverse) inverse[i] = v;
    }
    return MOE_OK;
}

double moe_profile_hit_rate(const uint16_t* pairs, int n_pairs, int L, int E, int slots, const uint32_t* hist) {
    if (!hist || (!pairs && n_pairs > 0) || L < 1 || E < 1 || n_pairs < 0 || slots < 0) return -1.0;
    const int use = std::min(slots, n_pairs);
    uint64_t total = 0, hit = 0;
    for (int64_t i = 0; i < (int64_t)L * E; ++i) total += hist[i];
    std::vector<char> cached((size_t)L * E, 0);
    for (int r = 0; r < use; ++r) {
        const int l = pairs[2 * r], e = pairs[2 * r + 1];
        if (l >= L || e >= E) return -1.0;
        const size_t i = (size_t)l * E + e;
        if (!cached[i]) hit += hist[i];
        cached[i] = 1;
    }
    return total ? (double)hit / (double)total : 0.0;
}

int moe_last_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_moe_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_moe_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

int moe_set_stage_events(void* const* events, int n) {
    if (n < 0 || (n > 0 && !events)) return MOE_ERR_ARG;
    std::lock_guard<std::mutex> g(g_mu);
    g_stage_ev.clear();
    for (int i = 0; i < n; ++i) g_stage_ev.push_back(static_cast<cudaEvent_t>(events[i]));
    return MOE_OK;
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

int moe_debug_set(int key, int value) {
    if (value < 0) return MOE_ERR_RANGE;
    switch (key) {
        case MOE_DBG_SPIN_LIMIT: g_dbg_spin = (unsigned)value; return MOE_OK;
        case MOE_DBG_BARRIER_EXTRA: g_dbg_bar1 = (unsigned)value; return MOE_OK;
        default: return MOE_ERR_ARG;
    }
}

size_t moe_workspace_offset(int T, int E, int top_k, int H, int I, int field) {
    if (T < 1 || E < 1 || top_k < 1 || H < 1 || I < 1) return (size_t)-1;
    const Ws L = ws_layout(T, E, top_k, H, I);
    switch (field) {
        case MOE_WS_FAST_LOGITS: return L.logit;
        case MOE_WS_PAIR_OUT: return L.y;
        case MOE_WS_SLOW_COUNT: return L.slow;
        default: return (size_t)-1;
    }
}

double moe_router_gamma(int T, int E, int H) {
    if (T <= MOE_DECODE_MAX_T || E < 1 || E > MOE_MAX_E || H < 32 || H % 32) return -1.0;
    if (T <= MOE_ROUTER_F64_MAX_T) return (double)(H + 32) * 1.1102230246251565e-16 * 1.01;  // fp64 tensor cores
    if (E % RT_BM == 0 && H % RT_BK == 0) return moe_tc_router_gamma(H);  // tensor-core chunk router
    return gamma_n(RG_BK + H / RG_BK + 2, 5.9604644775390625e-8);      // CUDA-core chunk router
}

int moe_timeout_site(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_moe_where, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_moe_where, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

#ifdef MOE_PROBE
// Measurement builds only: the fused decode kernel's phase timestamps of the last launch.
int moe_probe_read(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_df_probe, sizeof(g_df_probe)) == cudaSuccess ? 0 : -1;
}
int moe_probe_warps(unsigned long long* host, int clear) {
    if (cudaMemcpyFromSymbol(host, g_df_wprobe, sizeof(g_df_wprobe)) != cudaSuccess) return -1;
    if (clear) {
        static unsigned long long zero[160 * DF_WARPS_PROBE * DF_NWP];
        if (cudaMemcpyToSymbol(g_df_wprobe, zero, sizeof(zero)) != cudaSuccess) return -1;
    }
    return 0;
}
#endif

const char* moe_strerror(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument: null, misaligned or overlapping pointer";
        case MOE_ERR_SHAPE: return "unsupported shape: H, I, block, bit width or arena layout";
        case MOE_ERR_RANGE: return "value out of range: T, E, top_k, L or layer";
        case MOE_ERR_WS: return "workspace smaller than moe_workspace_bytes()";
        case MOE_ERR_CUDA: return "CUDA launch or query failed";
        case MOE_ERR_SLOT: return "a selected expert has no valid arena slot (it contributed zero)";
        case MOE_ERR_TIMEOUT: return "a bounded device-side wait expired";
        case MOE_ERR_STATIC: return "size beyond the fixed scratch of moe_route_static (T > MOE_ROUTE_STATIC_MAX_T)";
        default: return "unknown error code";
    }
}

}  // extern "C"
