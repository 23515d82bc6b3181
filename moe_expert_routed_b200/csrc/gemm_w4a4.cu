// gemm_w4a4.cu -- W4A4 on the tensor cores: NVFP4 weights times NVFP4 activations
// with the block-scaled MMA (tcgen05.mma kind::mxf4nvf4, one E4M3 factor per 16
// values of each operand, fp32 accumulators in TMEM).
//
// The operation is the sum over j of w[e][col][j] * x^[t][j], with w the NVFP4
// weight (e2m1 code * E4M3 block scale * scale2[e]) and x^ the NVFP4 activation
// (e2m1 code * E4M3 block scale * g[t], see actq.cu). The MMA forms the products
// e2m1 * e2m1 * s_w * s_x exactly and sums them in fp32; the epilogue multiplies by
// scale2[e] and g[t] (the weights' second-level scale, spark_model helpers_a.rs,
// and the activations' per-token scale).
//
// Work items as in the bf16 grouped GEMM: (tile of up to 128 pairs of one expert,
// 128 weight rows), claimed by a persistent grid. A k-tile is 256 values: one
// 128-byte row of packed codes per weight row and per pair, four MMAs of K = 64.
// Warp roles (608 threads):
//   warps 0-7   block-scale writers: per k-tile, warps 0-3 move the weight rows'
//               E4M3 factors and warps 4-7 the pairs' from the stage into tensor
//               memory (tcgen05.st), in the layout the MMA reads: for each K = 64
//               block, 4 columns, lane L of column c holding the 4 factors of row
//               (L mod 32) + 32 c (every quarter of the lanes holds the same words);
//               then they publish the stage
//   warps 8-11  loaders: cp.async of the pairs' activation codes (128 bytes per pair
//               and k-tile) into the B tile, 128-byte swizzle, and of their 16 factor
//               bytes
//   warp 12     TMEM allocation; one lane issues the MMAs and commits
//   warp 13     one lane: the weight codes of each k-tile as two 64-row 2-D TMA boxes
//               (128-byte swizzle, no multicast) straight into the A tile, and the
//               rows' factors as one 128-row box
//   warps 14-17 epilogue: TMEM -> registers, x scale2[e] x g[t], one rounding, row p
//   warp 18     scheduler
// Every wait is bounded (1 s); a wait that gives up sets ERR_TIMEOUT, and the CTA
// lets its copies and MMAs in flight complete before freeing TMEM and exiting.
#include <string.h>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr uint32_t W4_BM = 128, W4_BN = 128, W4_KT = 256;    // weight rows, pairs, values per k-tile
constexpr uint32_t W4_TILE = 128u * 128u;                     // bytes of an A or B tile (128 rows x 128 B)
constexpr uint32_t W4_SFT = 128u * 16u;                       // a tile's E4M3 factors: 128 rows x 16 bytes
// stage: A codes, B codes, A factors, B factors (row r's 16 factor bytes at 16 r)
constexpr uint32_t W4_STAGE = 2u * W4_TILE + 2u * W4_SFT;
constexpr uint32_t W4_MAX_STAGES = 6;
constexpr int W4_THREADS = 608;
constexpr int W4_LD_WARP0 = 8, W4_MMA_WARP = 12, W4_TMA_WARP = 13, W4_EPI_WARP0 = 14, W4_SCHED_WARP = 18;
constexpr uint32_t W4_RING = 4;
constexpr uint32_t W4_RING_READERS = 8 + 4 + 4 + 2;  // writer, loader, epilogue warps; MMA and TMA lanes
constexpr uint32_t W4_ACC_COLS = 2u * W4_BN;          // two accumulators
constexpr uint32_t W4_SF_COLS = 32;                   // per stage: 16 for A's factors, 16 for B's
constexpr uint64_t W4_WAIT_NS = 1000000000ull;
static_assert(W4_EPI_WARP0 + 4 == W4_SCHED_WARP && W4_SCHED_WARP * 32 + 32 == W4_THREADS, "warp roles");

struct W4Params {
    const uint8_t *wcodes;       // [E * n][k / 2] packed E2M1 (through the tensor map)
    const uint8_t *wscales;      // [E * n][k / 16] E4M3
    const float *scale2;         // [E]
    const uint8_t *xcodes;       // [m][k / 2]
    const uint8_t *xscales;      // [m][k / 16]
    const float *gscale;         // [m]
    const uint32_t *offsets, *sorted_pairs, *tiles, *tile_count;
    uint32_t *work_counter;
    void *out;
    uint32_t *err;
    uint32_t k, n, n_expert_used, ktiles, n_mtiles, stages;
    int out_dtype;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint32_t w4_swz(uint32_t r, uint32_t c) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4);
}

__global__ void __launch_bounds__(W4_THREADS, 1)
gemm_w4a4_kernel(const W4Params P, const __grid_constant__ CUtensorMap wmap,
                 const __grid_constant__ CUtensorMap smap) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[3 * W4_MAX_STAGES + 6 + 2 * W4_RING];
    __shared__ uint32_t ring_s[W4_RING];
    __shared__ uint32_t tmem_s;
    __shared__ int abort_s;

    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t S = P.stages;
    const uint32_t nm = P.n_mtiles;
    const uint32_t n_items = __ldg(P.tile_count) * nm;
    const uint32_t base = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t full0 = ptx::smem_u32(&bars[0]);
    const uint32_t loaded0 = ptx::smem_u32(&bars[W4_MAX_STAGES]);
    const uint32_t empty0 = ptx::smem_u32(&bars[2 * W4_MAX_STAGES]);
    const uint32_t accfull0 = ptx::smem_u32(&bars[3 * W4_MAX_STAGES]);
    const uint32_t accempty0 = ptx::smem_u32(&bars[3 * W4_MAX_STAGES + 2]);
    const uint32_t drainb = ptx::smem_u32(&bars[3 * W4_MAX_STAGES + 4]);
    const uint32_t ringfull0 = ptx::smem_u32(&bars[3 * W4_MAX_STAGES + 6]);
    const uint32_t ringempty0 = ptx::smem_u32(&bars[3 * W4_MAX_STAGES + 6 + W4_RING]);
    volatile int *abort_flag = &abort_s;
    volatile uint32_t *ring = ring_s;
    const uint32_t kb16 = P.k / 16u;  // factor bytes per row

    auto wait = [&](uint32_t bar, uint32_t par) -> bool {
        return ptx::mbar_wait_bounded(bar, par, abort_flag, P.err, ERR_TIMEOUT, P.timeout_ns);
    };
    auto next_item = [&](uint32_t i, bool whole_warp, uint32_t &w) -> bool {
        const uint32_t slot = i % W4_RING;
        if (!wait(ringfull0 + 8 * slot, (i / W4_RING) & 1u)) return false;
        w = ring[slot];
        if (whole_warp) __syncwarp();
        if (!whole_warp || lane == 0) ptx::mbar_arrive(ringempty0 + 8 * slot);
        return true;
    };
    // item w: tile w / nm (expert e, first pair r0: pairs off + r0 .. + nt - 1), rows row0 ..
    struct It {
        uint32_t e, r0, off, nt, nt_pad, row0;
    };
    auto load_item = [&](uint32_t w) -> It {
        It it;
        const uint32_t t = w / nm;
        it.e = __ldg(P.tiles + 2 * t);
        it.r0 = __ldg(P.tiles + 2 * t + 1);
        it.off = __ldg(P.offsets + it.e);
        const uint32_t cnt = __ldg(P.offsets + it.e + 1) - it.off;
        it.nt = tmin<uint32_t>(W4_BN, cnt - it.r0);
        it.nt_pad = (it.nt + 15u) & ~15u;
        it.row0 = (w % nm) * W4_BM;
        return it;
    };

    if (tid == 0) {
        for (uint32_t s = 0; s < S; s++) {
            ptx::mbar_init(full0 + 8 * s, 256);      // the block-scale writers
            ptx::mbar_init(loaded0 + 8 * s, 128 + 1);  // the loaders and the tensor-copy lane
            ptx::mbar_init(empty0 + 8 * s, 1);
        }
        for (uint32_t b = 0; b < 2; b++) {
            ptx::mbar_init(accfull0 + 8 * b, 1);
            ptx::mbar_init(accempty0 + 8 * b, 4);
        }
        ptx::mbar_init(drainb, 1);
        for (uint32_t b = 0; b < W4_RING; b++) {
            ptx::mbar_init(ringfull0 + 8 * b, 1);
            ptx::mbar_init(ringempty0 + 8 * b, W4_RING_READERS);
        }
        ptx::fence_mbar_init();
        abort_s = 0;
    }
    if (warp == W4_MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(&tmem_s), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_s;

    if (warp < W4_LD_WARP0) {
        // ------------------------------------------------ block-scale writers
        const uint32_t opnd = warp >> 2, q = warp & 3u;  // 0: weights (A), 1: pairs (B)
        const uint32_t lanes = (32u * q) << 16;
        uint32_t g = 0;
        bool ok = true;
        for (uint32_t i = 0; ok; i++) {
            uint32_t w;
            if (!next_item(i, true, w) || w >= n_items) break;
            for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                const uint32_t s = g % S;
                if (!wait(loaded0 + 8 * s, (g / S) & 1u)) {
                    ok = false;
                    break;
                }
                // rows lane + 32 c of the tile: 16 factor bytes each, word a = K-block a's 4
                const uint8_t *sft = smem_raw + (base - ptx::smem_u32(smem_raw)) + s * W4_STAGE + 2u * W4_TILE +
                                     opnd * W4_SFT;
                uint4 f[4];
#pragma unroll
                for (int c = 0; c < 4; c++) f[c] = *(const uint4 *)(sft + 16u * (lane + 32u * c));
                uint32_t v[16];
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    v[0 + c] = f[c].x;
                    v[4 + c] = f[c].y;
                    v[8 + c] = f[c].z;
                    v[12 + c] = f[c].w;
                }
                ptx::tmem_st16(tmem + lanes + W4_ACC_COLS + W4_SF_COLS * s + 16u * opnd, v);
                ptx::tmem_wait_st();
                // the loaders' copies of this stage are visible to the MMAs' reads
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(full0 + 8 * s);
            }
        }
    } else if (warp < W4_MMA_WARP) {
        // ------------------------------------------------------------- loaders
        const uint32_t lt = tid - 256u;
        const uint32_t xc = lt & 7u, xi0 = lt >> 3;  // chunk, first row (rows xi0 + 16 j)
        const uint32_t rowb = P.k / 2u;             // code bytes per row
        uint32_t g = 0;
        bool ok = true;
        for (uint32_t i = 0; ok; i++) {
            uint32_t w;
            if (!next_item(i, true, w) || w >= n_items) break;
            const It it = load_item(w);
            const uint8_t *xrow[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const uint32_t r = xi0 + 16u * j;
                xrow[j] = r < it.nt ? P.xcodes + (size_t)(__ldg(P.sorted_pairs + it.off + it.r0 + r) /
                                                          P.n_expert_used) * rowb
                                    : nullptr;
            }
            // this thread's pair row lt: its factors
            const uint8_t *srow = lt < it.nt ? P.xscales + (size_t)(__ldg(P.sorted_pairs + it.off + it.r0 + lt) /
                                                                    P.n_expert_used) * kb16
                                             : nullptr;
            for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                const uint32_t s = g % S;
                if (g >= S && !wait(empty0 + 8 * s, ((g / S) - 1u) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t bt = base + s * W4_STAGE + W4_TILE;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const uint32_t r = xi0 + 16u * j;
                    if (r < it.nt_pad) {
                        const bool in = xrow[j] != nullptr;
                        const uint8_t *src = in ? xrow[j] + kt * 128u + xc * 16u : P.xcodes;
                        ptx::cp_async_16(bt + w4_swz(r, xc), src, in ? 16u : 0u);
                    }
                }
                ptx::cp_async_16(base + s * W4_STAGE + 2u * W4_TILE + W4_SFT + 16u * lt,
                                 srow ? srow + kt * 16u : P.xscales, srow ? 16u : 0u);
                ptx::cp_async_mbar_arrive(loaded0 + 8 * s);
            }
        }
        ptx::cp_async_wait_all();
    } else if (warp == W4_TMA_WARP) {
        // ------------------------------------------------------ weight codes
        if (lane == 0) {
            ptx::prefetch_tensormap(&wmap);
            ptx::prefetch_tensormap(&smap);
            uint32_t g = 0, last_s = 0, last_par = 0;
            bool any = false, ok = true;
            for (uint32_t i = 0; ok; i++) {
                uint32_t w;
                if (!next_item(i, false, w) || w >= n_items) break;
                const It it = load_item(w);
                const int32_t y0 = (int32_t)(it.e * P.n + it.row0);
                for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                    const uint32_t s = g % S;
                    if (g >= S && !wait(empty0 + 8 * s, ((g / S) - 1u) & 1u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = loaded0 + 8 * s, at = base + s * W4_STAGE;
                    ptx::mbar_arrive_expect_tx(bar, W4_TILE + W4_SFT);
                    ptx::tma_load_2d(at, &wmap, (int32_t)(kt * 128u), y0, bar);
                    ptx::tma_load_2d(at + W4_TILE / 2u, &wmap, (int32_t)(kt * 128u), y0 + 64, bar);
                    ptx::tma_load_2d(at + 2u * W4_TILE, &smap, (int32_t)(kt * 16u), y0, bar);
                    last_s = s;
                    last_par = (g / S) & 1u;
                    any = true;
                }
            }
            if (any) ptx::mbar_wait_bounded(loaded0 + 8 * last_s, last_par, nullptr, P.err, ERR_TIMEOUT, W4_WAIT_NS);
        }
        __syncwarp();
    } else if (warp == W4_MMA_WARP) {
        // --------------------------------------------------------------- MMAs
        if (lane == 0) {
            bool ok = true;
            uint32_t g = 0, done = 0;
            for (uint32_t i = 0; ok; i++) {
                uint32_t w;
                if (!next_item(i, false, w)) {
                    ok = false;
                    break;
                }
                if (w >= n_items) break;
                const It it = load_item(w);
                const uint32_t buf = done % 2u, use = done / 2u;
                if (!wait(accempty0 + 8 * buf, (use & 1u) ^ 1u)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem + buf * W4_BN;
                const uint32_t idesc = ptx::idesc_nvf4(it.nt_pad);
                uint32_t accum = 0;
                for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                    const uint32_t s = g % S;
                    if (!wait(full0 + 8 * s, (g / S) & 1u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t at = base + s * W4_STAGE, bt = at + W4_TILE;
                    const uint32_t sf = tmem + W4_ACC_COLS + W4_SF_COLS * s;
#pragma unroll
                    for (uint32_t kb = 0; kb < 4; kb++) {
                        ptx::mma_nvf4_ss(d, ptx::sdesc_k128(at + 32u * kb), ptx::sdesc_k128(bt + 32u * kb), idesc,
                                         sf + 4u * kb, sf + 16u + 4u * kb, accum);
                        accum = 1;
                    }
                    ptx::mma_commit(empty0 + 8 * s);
                }
                if (!ok) break;
                ptx::mma_commit(accfull0 + 8 * buf);
                done++;
            }
            ptx::mma_commit(drainb);
            ptx::mbar_wait_bounded(drainb, 0, nullptr, P.err, ERR_TIMEOUT, W4_WAIT_NS);
        }
        __syncwarp();
    } else if (warp == W4_SCHED_WARP) {
        // ------------------------------------------------------------ scheduler
        if (lane == 0) {
            for (uint32_t i = 0;; i++) {
                const uint32_t slot = i % W4_RING;
                if (i >= W4_RING && !wait(ringempty0 + 8 * slot, ((i / W4_RING) - 1u) & 1u)) break;
                uint32_t w = i == 0 ? blockIdx.x : gridDim.x + atomicAdd(P.work_counter, 1u);
                if (w > n_items) w = n_items;
                ring[slot] = w;
                ptx::mbar_arrive(ringfull0 + 8 * slot);
                if (w >= n_items) break;
            }
        }
    } else {
        // ------------------------------------------------------------- epilogue
        const uint32_t q = warp & 3u;
        uint32_t done = 0;
        for (uint32_t i = 0;; i++) {
            uint32_t w;
            if (!next_item(i, true, w) || w >= n_items) break;
            const It it = load_item(w);
            const uint32_t buf = done % 2u, use = done / 2u;
            if (!wait(accfull0 + 8 * buf, use & 1u)) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + buf * W4_BN;
            const uint32_t row = it.row0 + q * 32u + lane;
            const float s2 = __ldg(P.scale2 + it.e);
            const uint32_t *pairs = P.sorted_pairs + it.off + it.r0;
            for (uint32_t c0 = 0; c0 < it.nt; c0 += 16) {
                uint32_t v[16], pr[16];
                float f[16];
                ptx::tmem_ld16(d + ((q * 32u) << 16) + c0, v);
                // lane j < 16 fetches column c0 + j's pair and its factor g[t] * scale2[e];
                // the warp shares them by shuffles
                const uint32_t cj = c0 + (lane & 15u);
                const uint32_t myp = cj < it.nt ? __ldg(pairs + cj) : 0u;
                const float myf = __ldg(P.gscale + myp / P.n_expert_used) * s2;
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    pr[j] = __shfl_sync(0xFFFFFFFFu, myp, j);
                    f[j] = __shfl_sync(0xFFFFFFFFu, myf, j);
                }
                ptx::tmem_wait_ld();
                if (row < P.n) {
                    const uint32_t nc = tmin<uint32_t>(16u, it.nt - c0);
                    if (P.out_dtype == DT_BF16) {
#pragma unroll
                        for (int j = 0; j < 16; j++)
                            if ((uint32_t)j < nc)
                                ((__nv_bfloat16 *)P.out)[(size_t)pr[j] * P.n + row] =
                                    __float2bfloat16_rn(__uint_as_float(v[j]) * f[j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; j++)
                            if ((uint32_t)j < nc)
                                store_out(P.out, P.out_dtype, (size_t)pr[j] * P.n + row, __uint_as_float(v[j]) * f[j]);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(accempty0 + 8 * buf);
            done++;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == W4_MMA_WARP) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 w4_encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return (PFN_cuTensorMapEncodeTiled_v12000)f;
    }();
    return fn;
}

uint32_t w4_sm_count() {
    static int count[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148u;
    if (count[dev] == 0) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
        count[dev] = c;
    }
    return (uint32_t)count[dev];
}

}  // namespace

bool w4a4_mma_supported(const QmmArgs &a) {
    return a.fmt == FMT_NVFP4 && !a.packed_ptrs && a.act < 0 && !a.bias && a.k % W4_KT == 0 && a.n > 0 &&
           (uintptr_t)a.packed % 16u == 0 && a.num_experts <= ROUTE_MAX_E &&
           (uint64_t)a.num_experts * a.n < (1ull << 31);
}

cudaError_t launch_gemm_w4a4(const QmmArgs &a, const uint8_t *xcodes, const uint8_t *xscales, const float *gscale,
                             const uint32_t *offsets, const uint32_t *sorted_pairs, const uint32_t *tiles,
                             const uint32_t *tile_count, uint32_t max_tiles, uint32_t *err, uint32_t *work_counter,
                             cudaStream_t st) {
    if (!w4a4_mma_supported(a)) return cudaErrorNotSupported;
    PFN_cuTensorMapEncodeTiled_v12000 enc = w4_encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap wmap;
    memset(&wmap, 0, sizeof(wmap));
    const cuuint64_t dims[2] = {a.k / 2u, (cuuint64_t)a.num_experts * a.n};
    const cuuint64_t strides[1] = {a.k / 2u};
    const cuuint32_t box[2] = {128u, 64u};
    const cuuint32_t estr[2] = {1u, 1u};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)a.packed, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorNotSupported;
    // the weight rows' E4M3 factors: [E * n, k / 16] bytes, boxes of 16 bytes x 128 rows
    CUtensorMap smap;
    memset(&smap, 0, sizeof(smap));
    const cuuint64_t sdims[2] = {a.k / 16u, (cuuint64_t)a.num_experts * a.n};
    const cuuint64_t sstrides[1] = {a.k / 16u};
    const cuuint32_t sbox[2] = {16u, 128u};
    if ((uintptr_t)a.scales % 16u != 0 ||
        enc(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)a.scales, sdims, sstrides, sbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorNotSupported;
    W4Params P{};
    P.wcodes = a.packed;
    P.wscales = (const uint8_t *)a.scales;
    P.scale2 = (const float *)a.aux;
    P.xcodes = xcodes;
    P.xscales = xscales;
    P.gscale = gscale;
    P.offsets = offsets;
    P.sorted_pairs = sorted_pairs;
    P.tiles = tiles;
    P.tile_count = tile_count;
    P.work_counter = work_counter;
    P.out = a.out;
    P.err = err;
    P.k = a.k;
    P.n = a.n;
    P.n_expert_used = a.n_expert_used;
    P.ktiles = a.k / W4_KT;
    P.n_mtiles = (a.n + W4_BM - 1) / W4_BM;
    P.out_dtype = a.out_dtype;
    P.timeout_ns = W4_WAIT_NS;
    // stages: 36 KB each (and 32 TMEM columns each beside the 256 of the accumulators)
    const size_t budget = 229000 - 1024;
    uint32_t S = (uint32_t)(budget / W4_STAGE);
    if (S > W4_MAX_STAGES) S = W4_MAX_STAGES;
    P.stages = S;
    const size_t smem = (size_t)S * W4_STAGE + 1024;
    static int smem_set[64];
    cudaError_t e = ensure_dyn_smem(gemm_w4a4_kernel, smem, smem_set);
    if (e != cudaSuccess) return e;
    const uint64_t items = (uint64_t)P.n_mtiles * max_tiles;
    const uint32_t ctas = (uint32_t)(items < (uint64_t)w4_sm_count() ? items : (uint64_t)w4_sm_count());
    gemm_w4a4_kernel<<<ctas, W4_THREADS, smem, st>>>(P, wmap, smap);
    return cudaGetLastError();
}

}  // namespace moe
