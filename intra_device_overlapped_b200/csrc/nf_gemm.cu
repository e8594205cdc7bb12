// Persistent bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by
// TMA, with the fused epilogues of the serving iteration.
//
//   C[M x N] = A[M x K] * B[N x K]^T,  A and B bf16 K-major, fp32 accumulation in TMEM.
//
// The iteration's projections (QKV, O, gate/up, down, LM head) are the
// compute-bound operations that NanoFlow keeps on the critical path while memory-
// bound attention of another nano-batch runs beside them (README "Introduction").
// Here each launch claims `grid` SMs: one CTA per SM (the 197 KB shared-memory
// footprint rules out a second resident CTA of any hot-path kernel), looping over
// 128 x 256 output tiles, either with a static stride or claimed one at a time from a
// global counter (GemmArgs::tile_ctr). With the counter, a launch of every SM made while
// another stream's kernel still holds some SMs runs on the free ones at once and grows onto
// the others as they are released: the GEMMs of one nano-batch take whatever share of the
// GPU the attention of another leaves.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: claims the next work unit and publishes it in a 4-entry
//               shared-memory ring read by the other roles; A box 128x64 and B box
//               256x64 per k-block into a 4-stage shared-memory ring (128-byte swizzle).
//   warp 1      TMEM allocator (512 columns = two 256-column accumulators) and the
//               single thread that issues tcgen05.mma (M=128, N=256, K=16) and
//               tcgen05.commit.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (thread = output row),
//               fused math, vectorised global stores. Double-buffered accumulators
//               let the epilogue of tile i run under the main loop of tile i+1.
// Every wait is bounded (NF_WAIT_LIMIT_NS); on timeout the CTA records
// NF_ERR_DEVICE_TIMEOUT, drains its outstanding copies and MMAs, frees TMEM, exits.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK, STAGES = kGemmStages;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t IDESC = umma_idesc_bf16_f32(BM, BN);

struct Tile {
    int a_row;      // TMA row of A
    int b_row;      // TMA row of B
    int row_begin;  // launch-row range covered by this tile
    int row_end;
    int n_blk;
};

__device__ __forceinline__ int total_tiles(const GemmArgs& p) {
    if (!p.grouped) return p.m_tiles * p.n_tiles;
    int t = 0;
    for (int g = 0; g < p.num_groups; ++g) {
        const int rows = p.group_offsets[g + 1] - p.group_offsets[g];
        t += ((rows + BM - 1) / BM) * p.n_tiles;
    }
    return t;
}

__device__ __forceinline__ Tile tile_at(const GemmArgs& p, int tile) {
    Tile t;
    if (!p.grouped) {
        const int mb = tile % p.m_tiles;
        t.n_blk = tile / p.m_tiles;
        t.row_begin = mb * BM;
        t.row_end = min(p.M, t.row_begin + BM);
        t.a_row = p.a_row0 + t.row_begin;
        t.b_row = t.n_blk * BN;
        return t;
    }
    int base = 0;
    for (int g = 0; g < p.num_groups; ++g) {
        const int r0 = p.group_offsets[g], r1 = p.group_offsets[g + 1];
        const int mt = (r1 - r0 + BM - 1) / BM;
        const int cnt = mt * p.n_tiles;
        if (tile < base + cnt) {
            const int local = tile - base;
            const int mb = local % mt;
            t.n_blk = local / mt;
            t.row_begin = r0 + mb * BM;
            t.row_end = min(r1, t.row_begin + BM);
            t.a_row = p.a_row0 + t.row_begin;
            t.b_row = g * p.N + t.n_blk * BN;
            return t;
        }
        base += cnt;
    }
    t.n_blk = 0; t.row_begin = 0; t.row_end = 0; t.a_row = 0; t.b_row = 0;
    return t;
}

__device__ __forceinline__ float row_scale(const GemmArgs& p, int row) {
    if (p.partials == nullptr) return 1.0f;
    const float* pr = p.partials + (size_t)(p.tok0 + row) * p.n_part;
    float s = 0.f;
    for (int j = 0; j < p.n_part; ++j) s += pr[j];
    return rsqrtf(s * p.inv_dim + p.eps);
}

__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float* v) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        d[q] = w;
    }
}

__device__ __forceinline__ void store_f32x32(float* dst, const float* v) {
    float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// 32 consecutive columns [c0, c0 + 32) of row `slot` of (K|V = kv, head g) in a page of the
// physical KV layout: [K|V][64-column half][head][16 rows][8 chunks of 16 B], logical chunk c
// of row r stored at chunk c ^ (r & 7). c0 is a multiple of 32, so the columns stay in one half.
__device__ __forceinline__ void store_kv_row32(uint16_t* page, int kv, int g, int nkv, int d, int slot, int c0,
                                               const float* v) {
    const int halves = d / 64;
    uint16_t* rowp = page + (((size_t)kv * halves + (c0 >> 6)) * nkv + g) * 16 * 64 + (size_t)slot * 64;
    const int chunk0 = (c0 & 63) >> 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4*>(rowp + (((chunk0 + q) ^ (slot & 7)) << 3)) = w;
    }
}

// Per-warp staging of a 32 x 32 fp32 block of the accumulator. After tcgen05.ld lane l holds
// row l; global rows are contiguous along columns, so the block is turned around in shared
// memory: afterwards lane l serves column quad (l & 7) of rows 4 i + (l >> 3), i = 0..7, and
// eight lanes cover one 128-byte row segment (four rows per warp access instead of 32). The
// 16-byte chunks of a row are XOR-swizzled by the row so that the row-wise writes and the
// column-quad reads are both free of bank conflicts.
__device__ __forceinline__ void stage_rows32(float* stg, int lane, const float* v) {
    float4* s4 = reinterpret_cast<float4*>(stg) + lane * 8;
#pragma unroll
    for (int q = 0; q < 8; ++q) s4[q ^ (lane & 7)] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ float4 staged_quad(const float* stg, int r, int c4) {
    return reinterpret_cast<const float4*>(stg)[r * 8 + (c4 ^ (r & 7))];
}

__device__ __forceinline__ int ld_acquire_gpu(const int* ptr) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int* ptr, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

// Warp-uniform wait: every lane tests the phase; if it has not completed, lane 0 waits with
// the time limit and the outcome is shared.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          int lane) {
    if (__all_sync(0xffffffffu, mbar_test_wait(smem_u32(bar), parity))) return true;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ------------------------------------------------------------------ epilogues
// Residual epilogue of one warp's 32 rows (rows rbase .. rbase + 31 of the tile), through the
// warp's staging block so that every global access is row-contiguous:
//   publish != null (first k half of a split tile): the fp32 partial goes to the workspace;
//   otherwise h = (part + acc) + resid, written back to resid (fp32), to out_bf16 and, if set,
//   out_f32; the row's sum of squares over this column block goes to out_partials.
// The global reads of a 32-column block (residual, first-half partial) are issued together one
// block ahead of their use, so that their latency overlaps the previous block's work instead of
// being paid once per row behind that row's stores.
struct ResidCtx {
    const GemmArgs* p;
    const Tile* t;
    uint32_t tacc;
    int rbase, lane;
    float* stg;
    const float* part;
};

__device__ __forceinline__ void resid_load(const ResidCtx& c, int j, float4 (&r)[8], float4 (&w)[8]) {
    const GemmArgs& p = *c.p;
    const int n0 = c.t->n_blk * BN;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rt = c.rbase + 4 * i + (c.lane >> 3);
        const int col = 32 * j + 4 * (c.lane & 7);
        if (c.part != nullptr) w[i] = __ldcg(reinterpret_cast<const float4*>(c.part + (size_t)rt * BN + col));
        const int row = c.t->row_begin + rt;
        if (row < c.t->row_end)
            r[i] = __ldcg(reinterpret_cast<const float4*>(p.resid + (size_t)(p.tok0 + row) * p.N + n0 + col));
    }
}

__device__ __forceinline__ void resid_block(const ResidCtx& c, int j, const float4 (&r)[8], const float4 (&w)[8],
                                            float (&ss)[8]) {
    const GemmArgs& p = *c.p;
    const int n0 = c.t->n_blk * BN;
    float v[32];
    tmem_ld32(c.tacc + 32 * j, v);
    stage_rows32(c.stg, c.lane, v);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rt = c.rbase + 4 * i + (c.lane >> 3);
        const int col = 32 * j + 4 * (c.lane & 7);
        float4 x = staged_quad(c.stg, 4 * i + (c.lane >> 3), c.lane & 7);
        if (c.part != nullptr)  // split-K: first half's partial + this half, in that order
            x = make_float4(w[i].x + x.x, w[i].y + x.y, w[i].z + x.z, w[i].w + x.w);
        const int row = c.t->row_begin + rt;
        if (row < c.t->row_end) {
            const size_t g = (size_t)(p.tok0 + row);
            x = make_float4(x.x + r[i].x, x.y + r[i].y, x.z + r[i].z, x.w + r[i].w);
            ss[i] += x.x * x.x;
            ss[i] += x.y * x.y;
            ss[i] += x.z * x.z;
            ss[i] += x.w * x.w;
            *reinterpret_cast<float4*>(p.resid + g * p.N + n0 + col) = x;
            *reinterpret_cast<uint2*>(p.out_bf16 + g * p.ld_bf16 + n0 + col) =
                make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
            if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + g * p.ld_f32 + n0 + col) = x;
        }
    }
    __syncwarp();  // the next block overwrites the staging buffer
}

static_assert((BN / 32) % 2 == 0, "the residual epilogue walks column blocks in pairs");

__device__ __forceinline__ void epilogue_resid(const GemmArgs& p, const Tile& t, uint32_t tacc, int rbase, int lane,
                                               float* stg, const float* part, float* publish) {
    if (publish != nullptr) {
#pragma unroll 1
        for (int j = 0; j < BN / 32; ++j) {
            float v[32];
            tmem_ld32(tacc + 32 * j, v);
            stage_rows32(stg, lane, v);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int rt = rbase + 4 * i + (lane >> 3);
                __stcg(reinterpret_cast<float4*>(publish + (size_t)rt * BN + 32 * j + 4 * (lane & 7)),
                       staged_quad(stg, 4 * i + (lane >> 3), lane & 7));
            }
            __syncwarp();
        }
        return;
    }
    const ResidCtx c{&p, &t, tacc, rbase, lane, stg, part};
    float ss[8];
    float4 ra[8], wa[8], rb[8], wb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        ss[i] = 0.f;
        ra[i] = rb[i] = wa[i] = wb[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    resid_load(c, 0, ra, wa);
#pragma unroll 1
    for (int j = 0; j < BN / 32; j += 2) {
        resid_load(c, j + 1, rb, wb);
        resid_block(c, j, ra, wa, ss);
        if (j + 2 < BN / 32) resid_load(c, j + 2, ra, wa);
        resid_block(c, j + 1, rb, wb, ss);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float x = ss[i];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        const int row = t.row_begin + rbase + 4 * i + (lane >> 3);
        if ((lane & 7) == 0 && row < t.row_end) p.out_partials[(size_t)(p.tok0 + row) * p.n_tiles + t.n_blk] = x;
    }
}

// Each is called by all 32 lanes of an epilogue warp (tcgen05.ld is warp-collective);
// `valid` says whether this lane's row is inside the tile's row range.

template <int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& p, const Tile& t, uint32_t tacc, int row,
                                              bool valid) {
    float v[32];
    const int n0 = t.n_blk * BN;
    if constexpr (EPI == EPI_F32) {
        const float rs = valid ? row_scale(p, row) : 1.f;
        float* dst = p.out_f32 + (size_t)(p.tok0 + row) * p.ld_f32 + n0;
#pragma unroll 1
        for (int j = 0; j < BN / 32; ++j) {
            tmem_ld32(tacc + 32 * j, v);
            if (valid) {
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= rs;
                store_f32x32(dst + 32 * j, v);
            }
        }
    } else if constexpr (EPI == EPI_SWIGLU) {
        const float rs = valid ? row_scale(p, row) : 1.f;
        float u[32];
        uint16_t* dst = p.out_bf16 + (size_t)(p.tok0 + row) * p.ld_bf16 + t.n_blk * (BN / 2);
#pragma unroll 1
        for (int j = 0; j < BN / 64; ++j) {
            tmem_ld32(tacc + 32 * j, v);
            tmem_ld32(tacc + BN / 2 + 32 * j, u);
            if (valid) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float g = v[e] * rs;
                    const float up = u[e] * rs;
                    v[e] = g / (1.0f + __expf(-g)) * up;
                }
                store_bf16x32(dst + 32 * j, v);
            }
        }
    } else if constexpr (EPI == EPI_LMHEAD) {
        const float rs = valid ? row_scale(p, row) : 1.f;
        float best = -INFINITY;
        int arg = n0;
#pragma unroll 1
        for (int j = 0; j < BN / 32; ++j) {
            tmem_ld32(tacc + 32 * j, v);
            if (valid) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    v[e] *= rs;
                    if (v[e] > best) { best = v[e]; arg = n0 + 32 * j + e; }
                }
                if (p.out_bf16) store_bf16x32(p.out_bf16 + (size_t)(p.tok0 + row) * p.ld_bf16 + n0 + 32 * j, v);
            }
        }
        if (valid) {
            p.tile_max[(size_t)(p.tok0 + row) * p.n_tiles + t.n_blk] = best;
            p.tile_arg[(size_t)(p.tok0 + row) * p.n_tiles + t.n_blk] = arg;
        }
    } else if constexpr (EPI == EPI_QKV) {
        const int d = p.head_dim, half = d / 2;
        const int tok = p.tok0 + row;
        const float rs = valid ? row_scale(p, row) : 1.f;
        int pos = 0;
        long long page_base = -1;  // element offset of this token's page in the pool
        bool ok = valid;
        if (valid) {
            pos = p.positions[tok];
            if (pos < 0 || pos >= p.max_position) {
                set_status(p.status, NF_ERR_DEVICE_BOUNDS);
                ok = false;
            } else {
                const int req = tok < p.num_decode ? tok : p.num_decode;
                const int idx = p.page_indptr[req] + pos / 16;
                const int page = (idx < p.page_indptr[req + 1]) ? p.page_indices[idx] : -1;
                if (page < 0 || page >= p.num_pages) {
                    set_status(p.status, NF_ERR_DEVICE_BOUNDS);
                } else {
                    page_base = (long long)page * 2 * p.nkv * 16 * d;
                }
            }
        }
        const int slot = pos & 15;
        // the rotation angles depend on the position and the column pair only: each column
        // block's cos / sin row segment is loaded once (16-byte loads) for both heads of the tile
        const bool any_rope = n0 / d < p.nq + p.nkv;
        float x2[32], cs[32], sn[32];
#pragma unroll 1
        for (int j = 0; j < half / 32; ++j) {
            if (ok && any_rope) {
                const float4* c4 = reinterpret_cast<const float4*>(p.rope_cos + (size_t)pos * half + 32 * j);
                const float4* s4 = reinterpret_cast<const float4*>(p.rope_sin + (size_t)pos * half + 32 * j);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 c = __ldg(c4 + q), sv = __ldg(s4 + q);
                    cs[4 * q] = c.x; cs[4 * q + 1] = c.y; cs[4 * q + 2] = c.z; cs[4 * q + 3] = c.w;
                    sn[4 * q] = sv.x; sn[4 * q + 1] = sv.y; sn[4 * q + 2] = sv.z; sn[4 * q + 3] = sv.w;
                }
            }
#pragma unroll 1
            for (int hc = 0; hc < BN / d; ++hc) {
                const int head = (n0 + hc * d) / d;
                const int kind = head < p.nq ? 0 : (head < p.nq + p.nkv ? 1 : 2);
                const int g = kind == 1 ? head - p.nq : head - p.nq - p.nkv;
                tmem_ld32(tacc + hc * d + 32 * j, v);
                tmem_ld32(tacc + hc * d + half + 32 * j, x2);
                if (!ok || (kind != 0 && page_base < 0)) continue;
                if (kind < 2) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float a = v[e] * rs, b = x2[e] * rs;
                        v[e] = a * cs[e] - b * sn[e];
                        x2[e] = b * cs[e] + a * sn[e];
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) { v[e] *= rs; x2[e] *= rs; }
                }
                if (kind == 0) {
                    uint16_t* dst = p.q_out + ((size_t)tok * p.nq + head) * d;
                    store_bf16x32(dst + 32 * j, v);
                    store_bf16x32(dst + half + 32 * j, x2);
                } else {
                    store_kv_row32(p.kv_pool + page_base, kind - 1, g, p.nkv, d, slot, 32 * j, v);
                    store_kv_row32(p.kv_pool + page_base, kind - 1, g, p.nkv, d, slot, half + 32 * j, x2);
                }
            }
        }
    }
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // barriers in the kGemmBarrierBytes after the ring, then the epilogue warps' staging blocks
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;   // [2]
    uint64_t* tempty = tfull + 2;       // [2]
    uint64_t* drain = tempty + 2;       // [1]
    uint64_t* unit_full = drain + 1;    // [4] work-unit ring: published by the producer
    uint64_t* unit_empty = unit_full + 4;  // [4] read by the MMA warp and the four epilogue warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_empty + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* unit_ring = reinterpret_cast<volatile int*>(abort_flag + 1);  // [4], -1 = no more work

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint64_t t_start = 0;
    if (threadIdx.x == 0) {
        t_start = globaltimer_ns();
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 4); }
        mbar_init(drain, 1);
        for (int u = 0; u < 4; ++u) { mbar_init(&unit_full[u], 1); mbar_init(&unit_empty[u], 5); }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ntiles = total_tiles(p);
    const int ks = (EPI == EPI_RESID && p.k_split == 2) ? 2 : 1;  // k halves per tile
    const int nunits = ntiles * ks;
    const int kb_per = p.k_blocks / ks;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer. A (activations) is re-read by every column block: keep
            // it in L2 over the KV pages that attention streams beside this GEMM.
            const uint64_t a_policy = l2_policy_evict_last();
            uint32_t stage = 0, phase = 0;
            int pending[STAGES];
            for (int s = 0; s < STAGES; ++s) pending[s] = -1;  // parity of an unconsumed load, -1 = none
            bool ok = true;
            // units are claimed in increasing order; with the counter, the next claim is made while
            // the last k blocks of the current unit are loaded, so its latency stays hidden
            int next = p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : (int)blockIdx.x;
            for (int local = 0; ok; ++local) {
                const int unit = next < nunits ? next : -1;
                const int slot = local & 3;
                if (!mbar_wait(&unit_empty[slot], ((uint32_t)(local >> 2) & 1u) ^ 1u, abort_flag, p.status)) break;
                unit_ring[slot] = unit;
                mbar_arrive(&unit_full[slot]);
                if (unit < 0) break;
                const Tile t = tile_at(p, unit % ntiles);
                const int kb0 = (unit / ntiles) * kb_per;
                for (int kb = kb0; kb < kb0 + kb_per; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
                    pending[stage] = -1;
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    tma_load_2d_hint(sa, &tmA, &full[stage], kb * BK, t.a_row, a_policy);
                    tma_load_2d(sb, &tmB, &full[stage], kb * BK, t.b_row);  // B maps hold 128-row boxes
                    tma_load_2d(sb + B_BYTES / 2, &tmB, &full[stage], kb * BK, t.b_row + BN / 2);
                    pending[stage] = (int)phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if (kb == kb0 + kb_per - 1 - (STAGES < kb_per ? STAGES : kb_per - 1))
                        next = p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : unit + (int)gridDim.x;
                }
            }
            if (!ok || *abort_flag) {
                // Let every copy still in flight land before the CTA exits.
                volatile int quiet = 0;
                for (int s = 0; s < STAGES; ++s)
                    if (pending[s] >= 0) mbar_wait(&full[s], (uint32_t)pending[s], &quiet, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: the whole warp follows the loop and one elected lane issues,
        // with the stage's descriptors offset by constants and the accumulate flags fixed per MMA,
        // so that issue keeps ahead of the tensor core
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        const uint64_t desc0 = umma_desc_sw128(smem_u32(smem));
        for (int local = 0; ok; ++local) {
            const int slot = local & 3;
            if (!wait_warp(&unit_full[slot], (uint32_t)(local >> 2) & 1u, abort_flag, p.status, lane)) break;
            const int unit = unit_ring[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&unit_empty[slot]);
            if (unit < 0) break;
            const int acc = local & 1;
            const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
            if (!wait_warp(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, lane)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
            const int kb0 = (unit / ntiles) * kb_per;
            for (int kb = kb0; kb < kb0 + kb_per; ++kb) {
                if (!wait_warp(&full[stage], phase, abort_flag, p.status, lane)) { ok = false; break; }
                tc_fence_after();
                const uint64_t adesc = desc0 + (uint64_t)((stage * STAGE_BYTES) >> 4);
                const uint64_t bdesc = adesc + (uint64_t)(A_BYTES >> 4);
                if (elect_one()) {
                    // advance 16 bf16 = 32 bytes along K inside the 128-byte swizzle atom
                    if (kb == kb0) umma_bf16_c<false>(d_tmem, adesc, bdesc, IDESC);
                    else umma_bf16_c<true>(d_tmem, adesc, bdesc, IDESC);
#pragma unroll
                    for (int k = 1; k < BK / 16; ++k)
                        umma_bf16_c<true>(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), IDESC);
                    umma_commit(&empty[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok) {
                if (elect_one()) umma_commit(&tfull[acc]);
                __syncwarp();
            }
        }
        // All MMAs issued by this warp have completed once `drain` flips.
        if (elect_one()) umma_commit(drain);
        __syncwarp();
        if (lane == 0) {
            volatile int quiet = 0;
            mbar_wait(drain, 0, &quiet, nullptr);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue warps 2..5; TMEM lane quarter = warp % 4
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        for (int local = 0;; ++local) {
            const int slot = local & 3;
            bool okw = wait_warp(&unit_full[slot], (uint32_t)(local >> 2) & 1u, abort_flag, p.status, lane);
            const int unit = okw ? unit_ring[slot] : -1;
            __syncwarp();
            if (lane == 0 && okw) mbar_arrive(&unit_empty[slot]);
            if (bar_red_or(1, 128, !okw)) break;  // every epilogue warp read the same unit
            if (unit < 0) break;
            const int acc = local & 1;
            const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            // all four epilogue warps leave together, so that none waits alone at barrier 1 below
            if (bar_red_or(1, 128, !ok)) break;
            tc_fence_after();
            const int tile = unit % ntiles;
            const Tile t = tile_at(p, tile);
            const int row = t.row_begin + row_in_tile;
            const bool valid = row < t.row_end;
            const uint32_t tacc = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            if constexpr (EPI == EPI_RESID) {
                float* stg = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES + kGemmBarrierBytes) + quarter * 1024;
                float* ws = p.splitk_ws + (size_t)tile * BM * BN;
                if (ks == 2 && unit < ntiles) {
                    // first half of the k blocks: publish the fp32 partial for the second half
                    epilogue_resid(p, t, tacc, quarter * 32, lane, stg, nullptr, ws);
                    __threadfence();
                    bar_sync_n(1, 128);
                    if (warp == 2 && lane == 0) st_release_gpu(p.splitk_flags + tile, p.splitk_epoch);
                } else {
                    if (ks == 2) {
                        // second half: wait (bounded) until the first half of this tile is published
                        if (warp == 2 && lane == 0) {
                            const uint64_t t0 = globaltimer_ns();
                            while (ld_acquire_gpu(p.splitk_flags + tile) != p.splitk_epoch) {
                                if (*abort_flag) break;
                                if (globaltimer_ns() - t0 > NF_WAIT_LIMIT_NS) {
                                    *abort_flag = 1;
                                    set_status(p.status, NF_ERR_DEVICE_TIMEOUT);
                                    break;
                                }
                                __nanosleep(128);
                            }
                        }
                        bar_sync_n(1, 128);
                    }
                    epilogue_resid(p, t, tacc, quarter * 32, lane, stg, ks == 2 ? ws : nullptr, nullptr);
                }
            } else {
                epilogue_tile<EPI>(p, t, tacc, row, valid);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
    if (threadIdx.x == 0 && p.trace != nullptr) {
        const int i = atomicAdd(p.trace_ctr, 1);
        if (i < p.trace_cap) {
            p.trace[i].kernel = NF_KERNEL_GEMM;
            p.trace[i].smid = (int32_t)smid();
            p.trace[i].t_start = t_start;
            p.trace[i].t_end = globaltimer_ns();
        }
    }
}

// ------------------------------------------------------------------ CTA-pair kernel
// The same GEMM on pairs of SMs (clusters of 2 CTAs) with the tcgen05 pair MMA: a work unit is a
// 256 x 256 output tile; CTA rank r loads rows [128 r, 128 r + 128) of the tile's A rows and of its
// B columns (N half), and rank 0 issues M = 256 MMAs that read both CTAs' shared memory, so each
// CTA stages 32 KB per k-block for 128 x 256 of output instead of 48 KB: at the tensor core's rate
// the shared-memory traffic (TMA writes + MMA operand reads) of one SM drops from about 190 to about
// 125 bytes per clock, under the bandwidth shared memory delivers. Each CTA's TMEM holds its 128
// rows of the two 256-column accumulators; the epilogues are the one-CTA kernel's, on each CTA's rows.
//
// Barriers: full[s] lives in rank 0 and counts both CTAs' TMA bytes (64 KB); empty[s] and tfull[a]
// exist in both CTAs and are completed by rank 0's multicast commits; tempty[a] lives in rank 0 and
// counts the eight epilogue warps of the pair; the work-unit ring is written by rank 0's producer
// into both CTAs and its slots are freed (in rank 0) by every reader of the pair.
constexpr int STAGES2 = kGemm2Stages;
constexpr uint32_t A2_BYTES = 128 * BK * 2;   // 16 KB: this CTA's A rows
constexpr uint32_t B2_BYTES = 128 * BK * 2;   // 16 KB: this CTA's half of the B tile
constexpr uint32_t STAGE2_BYTES = A2_BYTES + B2_BYTES;
constexpr uint32_t IDESC2 = umma_idesc_bf16_f32(256, BN);

__device__ __forceinline__ Tile tile_at2(const GemmArgs& p, int tile, uint32_t rank) {
    const int m2 = (p.M + 255) / 256;
    const int mb = tile % m2;
    Tile t;
    t.n_blk = tile / m2;
    t.row_begin = mb * 256 + (int)rank * 128;
    t.row_end = min(p.M, t.row_begin + 128);
    t.a_row = p.a_row0 + t.row_begin;
    t.b_row = t.n_blk * BN + (int)rank * 128;
    return t;
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES2 * STAGE2_BYTES);
    uint64_t* empty = full + STAGES2;
    uint64_t* tfull = empty + STAGES2;      // [2]
    uint64_t* tempty = tfull + 2;           // [2] (rank 0)
    uint64_t* drain = tempty + 2;           // [1] (rank 0)
    uint64_t* unit_full = drain + 1;        // [4]
    uint64_t* unit_empty = unit_full + 4;   // [4] (rank 0)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_empty + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* unit_ring = reinterpret_cast<volatile int*>(abort_flag + 1);  // [4], -1 = no more work

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    uint64_t t_start = 0;
    if (threadIdx.x == 0) {
        t_start = globaltimer_ns();
        for (int s = 0; s < STAGES2; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 8); }
        mbar_init(drain, 1);
        for (int u = 0; u < 4; ++u) { mbar_init(&unit_full[u], 1); mbar_init(&unit_empty[u], 10); }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers and TMEM exist before any cross-CTA access
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ntiles = ((p.M + 255) / 256) * p.n_tiles;
    const int ks = (EPI == EPI_RESID && p.k_split == 2) ? 2 : 1;
    const int nunits = ntiles * ks;
    const int kb_per = p.k_blocks / ks;
    const int cluster = (int)(blockIdx.x >> 1), nclusters = (int)(gridDim.x >> 1);
    // rank 0's copies of the barriers this CTA signals across the pair
    const uint32_t full0 = mapa_shared(smem_u32(full), 0);
    const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);
    const uint32_t unit_empty0 = mapa_shared(smem_u32(unit_empty), 0);
    const uint32_t ring1 = mapa_shared(smem_u32(const_cast<int*>(unit_ring)), 1);
    const uint32_t unit_full1 = mapa_shared(smem_u32(unit_full), 1);

    // every reader of a ring slot frees it in rank 0 (locally there, remotely from rank 1)
    auto unit_read = [&](int slot) {
        if (leader) mbar_arrive(&unit_empty[slot]);
        else mbar_arrive_cluster(unit_empty0 + 8u * (uint32_t)slot);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer of this CTA's A rows and B half
            // A (activations) is re-read by every column block: keep it in L2; B (weights) is shared by
            // the row blocks of a column block, which run at about the same time, under the default policy
            const uint64_t a_policy = l2_policy_evict_last();
            const uint64_t b_policy = l2_policy_evict_normal();
            uint32_t stage = 0, phase = 0;
            int pending[STAGES2];
            for (int s = 0; s < STAGES2; ++s) pending[s] = -1;
            bool ok = true;
            int next = leader ? (p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : cluster) : 0;
            for (int local = 0; ok; ++local) {
                const int slot = local & 3;
                int unit;
                if (leader) {
                    // claim and publish the pair's next unit in both CTAs' rings
                    if (!mbar_wait(&unit_empty[slot], ((uint32_t)(local >> 2) & 1u) ^ 1u, abort_flag, p.status)) break;
                    unit = next < nunits ? next : -1;
                    unit_ring[slot] = unit;
                    st_shared_cluster(ring1 + 4u * (uint32_t)slot, unit);
                    mbar_arrive(&unit_full[slot]);
                    mbar_arrive_cluster(unit_full1 + 8u * (uint32_t)slot);
                } else {
                    if (!mbar_wait_cluster(&unit_full[slot], (uint32_t)(local >> 2) & 1u, abort_flag, p.status)) break;
                    unit = unit_ring[slot];
                    unit_read(slot);
                }
                if (unit < 0) break;
                const Tile t = tile_at2(p, unit % ntiles, rank);
                const int kb0 = (unit / ntiles) * kb_per;
                for (int kb = kb0; kb < kb0 + kb_per; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
                    pending[stage] = -1;
                    uint8_t* sa = smem + stage * STAGE2_BYTES;
                    uint8_t* sb = sa + A2_BYTES;
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE2_BYTES);
                    const uint32_t fb = full0 + 8u * stage;
                    tma_load_2d_pair(sa, &tmA, fb, kb * BK, t.a_row, a_policy);
                    tma_load_2d_pair(sb, &tmB, fb, kb * BK, t.b_row, b_policy);
                    if (leader) pending[stage] = (int)phase;
                    if (++stage == STAGES2) { stage = 0; phase ^= 1u; }
                    if (leader && kb == kb0 + kb_per - 1 - (STAGES2 < kb_per ? STAGES2 : kb_per - 1))
                        next = p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : unit + nclusters;
                }
            }
            if (leader && (!ok || *abort_flag)) {
                volatile int quiet = 0;
                for (int s = 0; s < STAGES2; ++s)
                    if (pending[s] >= 0) mbar_wait(&full[s], (uint32_t)pending[s], &quiet, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (leader) {
            // ---------------- MMA issuer of the pair (rank 0)
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            const uint64_t desc0 = umma_desc_sw128(smem_u32(smem));
            for (int local = 0; ok; ++local) {
                const int slot = local & 3;
                if (!wait_warp(&unit_full[slot], (uint32_t)(local >> 2) & 1u, abort_flag, p.status, lane)) break;
                const int unit = unit_ring[slot];
                __syncwarp();
                if (lane == 0) mbar_arrive(&unit_empty[slot]);
                if (unit < 0) break;
                const int acc = local & 1;
                const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
                if (!wait_warp(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, lane)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                const int kb0 = (unit / ntiles) * kb_per;
                for (int kb = kb0; kb < kb0 + kb_per; ++kb) {
                    if (!wait_warp(&full[stage], phase, abort_flag, p.status, lane)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = desc0 + (uint64_t)((stage * STAGE2_BYTES) >> 4);
                    const uint64_t bdesc = adesc + (uint64_t)(A2_BYTES >> 4);
                    if (elect_one()) {
                        if (kb == kb0) umma_bf16_pair<false>(d_tmem, adesc, bdesc, IDESC2);
                        else umma_bf16_pair<true>(d_tmem, adesc, bdesc, IDESC2);
#pragma unroll
                        for (int k = 1; k < BK / 16; ++k)
                            umma_bf16_pair<true>(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), IDESC2);
                        umma_commit_pair(&empty[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES2) { stage = 0; phase ^= 1u; }
                }
                if (ok) {
                    if (elect_one()) umma_commit_pair(&tfull[acc], 0x3);
                    __syncwarp();
                }
            }
            if (elect_one()) umma_commit_pair(drain, 0x1);
            __syncwarp();
            if (lane == 0) {
                volatile int quiet = 0;
                mbar_wait(drain, 0, &quiet, nullptr);
            }
            __syncwarp();
        }
    } else {
        // ---------------- epilogue warps 2..5 of each CTA on the CTA's 128 rows of the tile
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        for (int local = 0;; ++local) {
            const int slot = local & 3;
            bool okw = lane == 0 ? mbar_wait_cluster(&unit_full[slot], (uint32_t)(local >> 2) & 1u, abort_flag,
                                                     p.status)
                                 : true;
            okw = __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
            const int unit = okw ? unit_ring[slot] : -1;
            __syncwarp();
            if (lane == 0 && okw) unit_read(slot);
            if (bar_red_or(1, 128, !okw)) break;
            if (unit < 0) break;
            const int acc = local & 1;
            const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait_cluster(&tfull[acc], acc_phase, abort_flag, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (bar_red_or(1, 128, !ok)) break;
            tc_fence_after();
            const int tile = unit % ntiles;
            const Tile t = tile_at2(p, tile, rank);
            const int row = t.row_begin + row_in_tile;
            const bool valid = row < t.row_end;
            const uint32_t tacc = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            if constexpr (EPI == EPI_RESID) {
                float* stg = reinterpret_cast<float*>(smem + STAGES2 * STAGE2_BYTES + kGemmBarrierBytes) + quarter * 1024;
                const int wslot = tile * 2 + (int)rank;
                float* ws = p.splitk_ws + (size_t)wslot * BM * BN;
                if (ks == 2 && unit < ntiles) {
                    epilogue_resid(p, t, tacc, quarter * 32, lane, stg, nullptr, ws);
                    __threadfence();
                    bar_sync_n(1, 128);
                    if (warp == 2 && lane == 0) st_release_gpu(p.splitk_flags + wslot, p.splitk_epoch);
                } else {
                    if (ks == 2) {
                        if (warp == 2 && lane == 0) {
                            const uint64_t t0 = globaltimer_ns();
                            while (ld_acquire_gpu(p.splitk_flags + wslot) != p.splitk_epoch) {
                                if (*abort_flag) break;
                                if (globaltimer_ns() - t0 > NF_WAIT_LIMIT_NS) {
                                    *abort_flag = 1;
                                    set_status(p.status, NF_ERR_DEVICE_TIMEOUT);
                                    break;
                                }
                                __nanosleep(128);
                            }
                        }
                        bar_sync_n(1, 128);
                    }
                    epilogue_resid(p, t, tacc, quarter * 32, lane, stg, ks == 2 ? ws : nullptr, nullptr);
                }
            } else {
                epilogue_tile<EPI>(p, t, tacc, row, valid);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(&tempty[acc]);
                else mbar_arrive_cluster(tempty0 + 8u * (uint32_t)acc);
            }
        }
        __syncwarp();
    }

    __syncthreads();
    tc_fence_before();
    cluster_sync_all();  // rank 0's MMAs into this CTA's TMEM and every cross-CTA arrive are done
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    if (threadIdx.x == 0 && p.trace != nullptr) {
        const int i = atomicAdd(p.trace_ctr, 1);
        if (i < p.trace_cap) {
            p.trace[i].kernel = NF_KERNEL_GEMM;
            p.trace[i].smid = (int32_t)smid();
            p.trace[i].t_start = t_start;
            p.trace[i].t_end = globaltimer_ns();
        }
    }
}

template <int EPI>
cudaError_t launch_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args, int grid,
                        cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm2_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kGemm2SmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    gemm2_kernel<EPI><<<grid, kGemmThreads, kGemm2SmemBytes, stream>>>(tmA, tmB, args);
    return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_one(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args, int grid,
                       cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kGemmSmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    gemm_kernel<EPI><<<grid, kGemmThreads, kGemmSmemBytes, stream>>>(tmA, tmB, args);
    return cudaGetLastError();
}

}  // namespace

bool gemm_uses_pairs(const GemmArgs& a) { return !a.grouped; }

int gemm_units(const GemmArgs& a) {
    const int ks = a.k_split == 2 ? 2 : 1;
    if (gemm_uses_pairs(a)) return ((a.M + 255) / 256) * a.n_tiles * ks;
    return a.m_tiles * a.n_tiles * ks;
}

cudaError_t launch_gemm(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args, int grid,
                        cudaStream_t stream) {
    if (grid <= 0) return cudaSuccess;
    if (gemm_uses_pairs(args) && grid >= 2) {
        const int g = grid & ~1;  // whole pairs
        switch (epi) {
            case EPI_F32: return launch_pair<EPI_F32>(tmA, tmB, args, g, stream);
            case EPI_QKV: return launch_pair<EPI_QKV>(tmA, tmB, args, g, stream);
            case EPI_RESID: return launch_pair<EPI_RESID>(tmA, tmB, args, g, stream);
            case EPI_SWIGLU: return launch_pair<EPI_SWIGLU>(tmA, tmB, args, g, stream);
            case EPI_LMHEAD: return launch_pair<EPI_LMHEAD>(tmA, tmB, args, g, stream);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (epi) {
        case EPI_F32: return launch_one<EPI_F32>(tmA, tmB, args, grid, stream);
        case EPI_QKV: return launch_one<EPI_QKV>(tmA, tmB, args, grid, stream);
        case EPI_RESID: return launch_one<EPI_RESID>(tmA, tmB, args, grid, stream);
        case EPI_SWIGLU: return launch_one<EPI_SWIGLU>(tmA, tmB, args, grid, stream);
        case EPI_LMHEAD: return launch_one<EPI_LMHEAD>(tmA, tmB, args, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace nf
