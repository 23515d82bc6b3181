// route.cu -- routing prologue of the grouped path: per-chunk expert histogram,
// exclusive scan, stable permutation of the (token, slot) pairs and the tile
// list. It produces the expert_offsets / sorted_token_ids pair that the routed
// grouped GEMM consumes (metrale helpers_b.rs, launch_grouped_gemm), here with a
// deterministic order: pairs of one expert stay in ascending pair index.
//
// Three launches, no inter-CTA waiting:
//   route_hist    one CTA per chunk of ROUTE_CHUNK ids: shared-memory histogram
//   route_scan    one CTA: bucket totals, offsets, per-(chunk, bucket) bases,
//                 tile list
//   route_scatter one CTA per chunk: per-warp bucket counts, their prefix over
//                 the warps, then stable ranks from warp match masks
// and, for the grouped GEMM with f32 x when the caller's workspace has room for it,
//   gather_x      the pairs' x rows in expert order (row i = x row of the token of
//                 sorted pair i) as bf16 high halves (rows 0 .. R-1) and the bf16
//                 roundings of the remainders (rows R .. 2R-1), so that the GEMM loads
//                 each tile of x rows with one tensor copy per half and no longer
//                 splits f32 values per tile (16-bit x needs no such pass: the GEMM
//                 gathers its rows with 4-row tensor copies)
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr uint32_t ROUTE_WARPS = ROUTE_THREADS / 32;
constexpr uint32_t ROUTE_PER_WARP = ROUTE_CHUNK / ROUTE_WARPS;  // ids per warp slice
constexpr uint32_t ROUTE_ROUNDS = ROUTE_PER_WARP / 32;          // ids per lane

// Bucket of each id of this warp's slice of the chunk (ids past R: ~0u), all
// loads issued before any is used. Lane l holds ids slice + 32 r + l.
__device__ __forceinline__ void load_buckets(const uint32_t *__restrict__ ids, uint32_t R, uint32_t E,
                                             uint32_t (&bk)[ROUTE_ROUNDS]) {
    const uint64_t w0 = (uint64_t)blockIdx.x * ROUTE_CHUNK + (threadIdx.x >> 5) * ROUTE_PER_WARP;
    const uint32_t lane = threadIdx.x & 31u;
#pragma unroll
    for (uint32_t r = 0; r < ROUTE_ROUNDS; r++) {
        const uint64_t i = w0 + 32u * r + lane;
        bk[r] = i < R ? __ldg(ids + i) : 0u;
    }
#pragma unroll
    for (uint32_t r = 0; r < ROUTE_ROUNDS; r++) {
        const uint64_t i = w0 + 32u * r + lane;
        bk[r] = i < R ? (bk[r] < E ? bk[r] : E) : 0xFFFFFFFFu;
    }
}

__global__ void __launch_bounds__(ROUTE_THREADS)
route_hist(const uint32_t *__restrict__ ids, uint32_t R, uint32_t E, uint32_t *__restrict__ chunk_hist) {
    extern __shared__ uint32_t hist[];
    const uint32_t NB = E + 1;
    uint32_t bk[ROUTE_ROUNDS];
    load_buckets(ids, R, E, bk);
    for (uint32_t b = threadIdx.x; b < NB; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31u;
#pragma unroll
    for (uint32_t r = 0; r < ROUTE_ROUNDS; r++) {
        // one atomic per distinct bucket of the warp's 32 ids
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bk[r]);
        if (bk[r] <= E && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&hist[bk[r]], (uint32_t)__popc(peers));
    }
    __syncthreads();
    for (uint32_t b = threadIdx.x; b < NB; b += blockDim.x)
        chunk_hist[(size_t)blockIdx.x * NB + b] = hist[b];
}

// Exclusive scan of one value per thread across the block (blockDim.x <= 1024,
// multiple of 32). `scratch` holds 33 words. Returns the exclusive prefix and the
// block total in *total.
__device__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *scratch, uint32_t *total) {
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        uint32_t t = __shfl_up_sync(0xFFFFFFFFu, inc, d);
        if (lane >= (uint32_t)d) inc += t;
    }
    if (lane == 31) scratch[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < nw ? scratch[lane] : 0u;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            uint32_t t = __shfl_up_sync(0xFFFFFFFFu, s, d);
            if (lane >= (uint32_t)d) s += t;
        }
        if (lane < nw) scratch[lane] = s - (lane < nw ? scratch[lane] : 0u);  // exclusive
        if (lane == nw - 1) scratch[32] = s;
    }
    __syncthreads();
    uint32_t res = scratch[warp] + inc - v;
    *total = scratch[32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(1024)
route_scan(const uint32_t *__restrict__ chunk_hist, uint32_t C, uint32_t E, uint32_t R,
           uint32_t tile_rows, uint32_t *__restrict__ counts, uint32_t *__restrict__ offsets,
           uint32_t *__restrict__ chunk_base, uint32_t *__restrict__ tiles,
           uint32_t *__restrict__ tile_count, uint32_t max_tiles, uint32_t *__restrict__ err,
           uint32_t *__restrict__ work_counter) {
    extern __shared__ uint32_t sm[];
    const uint32_t NB = E + 1;
    uint32_t *tot = sm;            // [NB]
    uint32_t *scratch = sm + NB;   // [33]
    for (uint32_t b = threadIdx.x; b < NB; b += blockDim.x) {
        uint32_t s = 0;
        for (uint32_t c = 0; c < C; c++) s += chunk_hist[(size_t)c * NB + b];
        tot[b] = s;
    }
    __syncthreads();
    // Each thread owns a contiguous segment of buckets.
    const uint32_t seg = (NB + blockDim.x - 1) / blockDim.x;
    const uint32_t b0 = min(threadIdx.x * seg, NB), b1 = min(b0 + seg, NB);
    uint32_t rows = 0, ntile = 0;
    for (uint32_t b = b0; b < b1; b++) {
        rows += tot[b];
        if (b < E) ntile += (tot[b] + tile_rows - 1) / tile_rows;
    }
    uint32_t total_rows, total_tiles;
    uint32_t row_off = block_exclusive_scan(rows, scratch, &total_rows);
    uint32_t tile_off = block_exclusive_scan(ntile, scratch, &total_tiles);
    for (uint32_t b = b0; b < b1; b++) {
        const uint32_t cnt = tot[b];
        counts[b] = cnt;
        offsets[b] = row_off;
        uint32_t run = row_off;
        for (uint32_t c = 0; c < C; c++) {
            chunk_base[(size_t)c * NB + b] = run;
            run += chunk_hist[(size_t)c * NB + b];
        }
        if (b < E) {
            for (uint32_t r0 = 0; r0 < cnt; r0 += tile_rows, tile_off++) {
                if (tile_off < max_tiles) {
                    tiles[2 * (size_t)tile_off] = b;
                    tiles[2 * (size_t)tile_off + 1] = r0;
                } else {
                    atomicOr(err, ERR_INTERNAL);
                }
            }
        }
        row_off += cnt;
    }
    if (threadIdx.x == 0) {
        offsets[NB] = total_rows;
        *tile_count = min(total_tiles, max_tiles);
        if (work_counter) *work_counter = 0u;  // the grouped GEMM's dynamic work counter
        if (total_rows != R) atomicOr(err, ERR_INTERNAL);
    }
}

// Stable scatter of one chunk. Each warp owns a contiguous slice of the chunk:
// pass 1 counts the slice's ids per bucket, then a per-bucket prefix over the
// warps (from the chunk's base) gives each warp its first position per bucket,
// and pass 2 walks the slice in order, ranking equal buckets inside each group
// of 32 ids by their match mask. Two block barriers in all.
__global__ void __launch_bounds__(ROUTE_THREADS)
route_scatter(const uint32_t *__restrict__ ids, uint32_t R, uint32_t E,
              const uint32_t *__restrict__ chunk_base, uint32_t *__restrict__ sorted_pairs,
              uint32_t *__restrict__ err, void *out, uint32_t n, int out_dtype) {
    extern __shared__ uint32_t wbase[];  // [ROUTE_WARPS][E + 1]
    const uint32_t NB = E + 1;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    uint32_t bk[ROUTE_ROUNDS];
    load_buckets(ids, R, E, bk);
    for (uint32_t b = tid; b < ROUTE_WARPS * NB; b += blockDim.x) wbase[b] = 0;
    __syncthreads();
    uint32_t *mine = wbase + warp * NB;
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (uint32_t r = 0; r < ROUTE_ROUNDS; r++) {
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bk[r]);
        if (bk[r] <= E && (peers & lt_mask) == 0) mine[bk[r]] += (uint32_t)__popc(peers);
        __syncwarp();
    }
    __syncthreads();
    for (uint32_t b = tid; b < NB; b += blockDim.x) {
        uint32_t run = chunk_base[(size_t)blockIdx.x * NB + b];
        for (uint32_t w = 0; w < ROUTE_WARPS; w++) {
            const uint32_t c = wbase[w * NB + b];
            wbase[w * NB + b] = run;
            run += c;
        }
    }
    __syncthreads();
    const uint64_t w0 = (uint64_t)blockIdx.x * ROUTE_CHUNK + warp * ROUTE_PER_WARP;
#pragma unroll
    for (uint32_t r = 0; r < ROUTE_ROUNDS; r++) {
        const uint32_t b = bk[r];
        const bool valid = b <= E;
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, b);
        const uint32_t i = (uint32_t)(w0 + 32u * r + lane);
        if (valid) {
            const uint32_t pos = mine[b] + (uint32_t)__popc(peers & lt_mask);
            if (pos < R) sorted_pairs[pos] = i;
            else atomicOr(err, ERR_INTERNAL);
            if (b == E) {
                atomicOr(err, ERR_BAD_ID);
                if (out)
                    for (uint32_t col = 0; col < n; col++) store_out(out, out_dtype, (size_t)i * n + col, 0.f);
            }
        }
        __syncwarp();
        if (valid && (peers & lt_mask) == 0) mine[b] += (uint32_t)__popc(peers);
        __syncwarp();
    }
}

// One warp per gathered row, 32-byte loads and 16-byte stores (k % 8 == 0). The split
// is the one the GEMM applies to f32 x it copies itself: hi = bf16(v), lo = bf16(v - hi),
// both rounded to nearest even.
__global__ void __launch_bounds__(256)
gather_x(const float *__restrict__ x, const uint32_t *__restrict__ sorted_pairs, uint32_t R, uint32_t k,
         uint32_t n_expert_used, uint16_t *__restrict__ xg) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t k8 = k / 8u;  // 8-element chunks per row
    for (uint32_t row = blockIdx.x * 8u + (threadIdx.x >> 5); row < R; row += gridDim.x * 8u) {
        const size_t t = __ldg(sorted_pairs + row) / n_expert_used;
        const float4 *src = (const float4 *)x + t * k8 * 2u;
        uint4 *hi = (uint4 *)xg + (size_t)row * k8, *lo = (uint4 *)xg + ((size_t)R + row) * k8;
        for (uint32_t c = lane; c < k8; c += 32u) {
            const float4 a = __ldg(src + 2u * c), b = __ldg(src + 2u * c + 1u);
            const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t h[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const __nv_bfloat162 hb = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
                const float2 hf = __bfloat1622float2(hb);
                const __nv_bfloat162 lb = __floats2bfloat162_rn(f[2 * i] - hf.x, f[2 * i + 1] - hf.y);
                h[i] = *reinterpret_cast<const uint32_t *>(&hb);
                l[i] = *reinterpret_cast<const uint32_t *>(&lb);
            }
            hi[c] = make_uint4(h[0], h[1], h[2], h[3]);
            lo[c] = make_uint4(l[0], l[1], l[2], l[3]);
        }
    }
}

// Per-token power of two for the f16 image of bf16 x: with a = max_j |x[t][j]| in
// [2^(E-1), 2^E), x * 2^(15-E) has its largest magnitude in [2^14, 2^15), inside f16's
// range, and a bf16 value (8 significant bits) times a power of two is exact in f16
// unless it falls below f16's normal range (2^-14, i.e. below 2^-28 of the token's
// largest). tok_scale[t] = 2^(E-15) undoes it in the GEMM's epilogue (1 for a zero row).
__global__ void __launch_bounds__(256)
x_token_scale(const uint16_t *__restrict__ x, uint32_t k, float *__restrict__ tok_scale) {
    __shared__ float red[8];
    const uint32_t t = blockIdx.x;
    float a = 0.f;
    for (uint32_t j = threadIdx.x; j < k; j += 256u) a = fmaxf(a, fabsf(bf16_bits_to_f32(__ldg(x + (size_t)t * k + j))));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, d));
    if ((threadIdx.x & 31u) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; w++) a = fmaxf(a, red[w]);
        const int e = a > 0.f ? ((int)((__float_as_uint(a) >> 23) & 0xFFu) - 126) : 15;  // a < 2^e
        const int s = e - 15 < -126 ? -126 : (e - 15 > 127 ? 127 : e - 15);
        tok_scale[t] = __uint_as_float((uint32_t)(s + 127) << 23);
    }
}

// The B operand image of the grouped GEMM: for tile t of the routing prologue's tile
// list and k-tile kt, rows 0 .. nt_pad-1 of the tile (its pairs' x rows; zeros past
// its pairs and past k) as f16, each row a 128-byte line with 16-byte chunk c at
// position c ^ (row & 7): block (t, kt) of bn lines starts at (t * ktiles + kt) * bn
// * 128 and is exactly the shared-memory tile (128-byte swizzle, K-major) the GEMM
// copies with one bulk copy. bf16 x is scaled per token by 1 / tok_scale; f16 x is
// copied. One warp per row, each lane a 16-byte chunk of 4 consecutive k-tiles.
__global__ void __launch_bounds__(256)
x_image(const uint16_t *__restrict__ x, int x_dtype, uint32_t k, uint32_t ktiles, const uint32_t *__restrict__ sp,
        const uint32_t *__restrict__ tiles, const uint32_t *__restrict__ tile_count,
        const uint32_t *__restrict__ offsets, uint32_t n_expert_used, uint32_t bn,
        const float *__restrict__ tok_scale, uint8_t *__restrict__ img) {
    const uint32_t t = blockIdx.x;
    if (t >= __ldg(tile_count)) return;
    const uint32_t e = __ldg(tiles + 2 * t), r0 = __ldg(tiles + 2 * t + 1);
    const uint32_t off = __ldg(offsets + e), cnt = __ldg(offsets + e + 1) - off;
    const uint32_t nt = cnt - r0 < bn ? cnt - r0 : bn, nt_pad = (nt + 15u) & ~15u;
    const uint32_t lane = threadIdx.x & 31u;
    for (uint32_t i = blockIdx.y * 8u + (threadIdx.x >> 5); i < nt_pad; i += gridDim.y * 8u) {
        const bool live = i < nt;
        const size_t tok = live ? __ldg(sp + off + r0 + i) / n_expert_used : 0;
        const uint16_t *xr = x + tok * k;
        float mul = 1.f;
        if (live && tok_scale) mul = 1.f / __ldg(tok_scale + tok);  // an exact power of two
#pragma unroll 4
        for (uint32_t q = lane; q < ktiles * 8u; q += 32u) {
            const uint32_t kt = q >> 3, c = q & 7u, j = kt * 64u + c * 8u;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (live && j < k) {
                v = __ldg((const uint4 *)(xr + j));
                if (x_dtype == DT_BF16) {
                    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int h = 0; h < 4; h++) {
                        const __half2 f = __floats2half2_rn(bf16_bits_to_f32(w[h] & 0xFFFFu) * mul,
                                                            bf16_bits_to_f32(w[h] >> 16) * mul);
                        w[h] = *reinterpret_cast<const uint32_t *>(&f);
                    }
                    v = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            uint8_t *line = img + (((size_t)t * ktiles + kt) * bn + i) * 128u;
            *(uint4 *)(line + ((c ^ (i & 7u)) << 4)) = v;
        }
    }
}

}  // namespace

cudaError_t launch_gather_x(const void *x, int x_dtype, const uint32_t *sorted_pairs, uint32_t R, uint32_t k,
                            uint32_t n_expert_used, uint16_t *xg, cudaStream_t st) {
    const uint32_t rows_per_cta = 8;
    uint32_t ctas = (R + rows_per_cta - 1) / rows_per_cta;
    if (ctas > 148u * 16u) ctas = 148u * 16u;
    if (ctas == 0) return cudaSuccess;
    if (x_dtype != DT_F32 || k % 8u != 0) return cudaErrorInvalidValue;
    gather_x<<<ctas, 256, 0, st>>>((const float *)x, sorted_pairs, R, k, n_expert_used, xg);
    return cudaGetLastError();
}

uint64_t x_image_bytes(uint64_t R, uint32_t E, uint32_t k, uint32_t tile_rows) {
    const uint64_t max_tiles = R / tile_rows + E + 1ull;
    return max_tiles * ((k + 63ull) / 64ull) * tile_rows * 128ull;
}

cudaError_t launch_x_image(const void *x, int x_dtype, uint32_t m, uint32_t k, const uint32_t *sorted_pairs,
                           const uint32_t *tiles, const uint32_t *tile_count, const uint32_t *offsets,
                           uint32_t n_expert_used, uint32_t tile_rows, uint32_t max_tiles, uint8_t *img,
                           float *tok_scale, cudaStream_t st) {
    if (x_dtype == DT_F32 || k % 8u != 0 || (tile_rows & 15u) || ((uintptr_t)x & 15u) || ((uintptr_t)img & 15u))
        return cudaErrorInvalidValue;
    const uint16_t *x16 = (const uint16_t *)x;
    if (x_dtype == DT_BF16) {
        if (!tok_scale) return cudaErrorInvalidValue;
        x_token_scale<<<m, 256, 0, st>>>(x16, k, tok_scale);
    } else {
        tok_scale = nullptr;
    }
    const uint32_t ktiles = (k + 63u) / 64u;
    const dim3 grid(max_tiles, (tile_rows + 31u) / 32u);
    x_image<<<grid, 256, 0, st>>>(x16, x_dtype, k, ktiles, sorted_pairs, tiles, tile_count, offsets, n_expert_used,
                                  tile_rows, tok_scale, img);
    return cudaGetLastError();
}

cudaError_t launch_route(const uint32_t *ids, uint32_t R, uint32_t E, uint32_t tile_rows,
                         uint32_t *counts, uint32_t *offsets, uint32_t *sorted_pairs,
                         uint32_t *tiles, uint32_t *tile_count, uint32_t max_tiles,
                         uint32_t *chunk_hist, uint32_t *chunk_base, uint32_t chunks,
                         uint32_t *err, void *out, uint32_t n, int out_dtype, cudaStream_t st,
                         uint32_t *work_counter) {
    const uint32_t NB = E + 1;
    route_hist<<<chunks, ROUTE_THREADS, NB * sizeof(uint32_t), st>>>(ids, R, E, chunk_hist);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    route_scan<<<1, 1024, (NB + 33) * sizeof(uint32_t), st>>>(
        chunk_hist, chunks, E, R, tile_rows, counts, offsets, chunk_base, tiles, tile_count,
        max_tiles, err, work_counter);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t sc_smem = (size_t)NB * ROUTE_WARPS * sizeof(uint32_t);
    route_scatter<<<chunks, ROUTE_THREADS, sc_smem, st>>>(ids, R, E, chunk_base, sorted_pairs,
                                                           err, out, n, out_dtype);
    return cudaGetLastError();
}

}  // namespace moe
