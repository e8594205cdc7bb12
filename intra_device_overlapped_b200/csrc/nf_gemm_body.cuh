// The one-CTA persistent GEMM on the 5th-generation tensor cores as a device function, with the fused
// epilogues of the serving iteration: shared by the GEMM kernels and by the persistent kernel that
// runs a whole layer (nf_mega.cu). The roles, tiles and waits are described in nf_gemm.cu.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace gemm_impl {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK, STAGES = kGemmStages;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t IDESC = umma_idesc_bf16_f32(BM, BN);
// mbarriers of the one-CTA body: full and empty per stage, tfull / tempty per accumulator, drain,
// unit_full / unit_empty per slot of the work-unit ring
constexpr int kBodyBarriers = 2 * STAGES + 2 + 2 + 1 + 4 + 4;

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
//   otherwise h = (part + acc) + resid, written back to resid (fp32) and to out_bf16; the row's
//   sum of squares over this column block goes to out_partials.
// The global reads of a 32-column block (residual, first-half partial) are issued together one
// block ahead of their use, so that their latency overlaps the previous block's work instead of
// being paid once per row behind that row's stores.
// The argument values the loops use are copied into the context once: the epilogue's global stores
// could alias the argument block where it is read through a pointer (not from the kernel's constant
// bank), which would make every store force a reload.
struct ResidCtx {
    float* resid;       // row 0 of the launch, column n0 of the tile
    uint16_t* out_bf16;
    int N, ld_bf16;
    int row_begin, row_end;
    uint32_t tacc;
    int rbase, lane;
    float* stg;
    const float* part;
};

__device__ __forceinline__ ResidCtx resid_ctx(const GemmArgs& p, const Tile& t, uint32_t tacc, int rbase, int lane,
                                              float* stg, const float* part) {
    const int n0 = t.n_blk * BN;
    ResidCtx c;
    c.resid = p.resid + (size_t)p.tok0 * p.N + n0;
    c.out_bf16 = p.out_bf16 + (size_t)p.tok0 * p.ld_bf16 + n0;
    c.N = p.N;
    c.ld_bf16 = p.ld_bf16;
    c.row_begin = t.row_begin;
    c.row_end = t.row_end;
    c.tacc = tacc;
    c.rbase = rbase;
    c.lane = lane;
    c.stg = stg;
    c.part = part;
    return c;
}

__device__ __forceinline__ void resid_load(const ResidCtx& c, int j, float4 (&r)[8], float4 (&w)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rt = c.rbase + 4 * i + (c.lane >> 3);
        const int col = 32 * j + 4 * (c.lane & 7);
        if (c.part != nullptr) w[i] = __ldcg(reinterpret_cast<const float4*>(c.part + (size_t)rt * BN + col));
        const int row = c.row_begin + rt;
        if (row < c.row_end) r[i] = __ldcg(reinterpret_cast<const float4*>(c.resid + (size_t)row * c.N + col));
    }
}

__device__ __forceinline__ void resid_block(const ResidCtx& c, int j, const float4 (&r)[8], const float4 (&w)[8],
                                            float (&ss)[8]) {
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
        const int row = c.row_begin + rt;
        if (row < c.row_end) {
            x = make_float4(x.x + r[i].x, x.y + r[i].y, x.z + r[i].z, x.w + r[i].w);
            ss[i] += x.x * x.x;
            ss[i] += x.y * x.y;
            ss[i] += x.z * x.z;
            ss[i] += x.w * x.w;
            *reinterpret_cast<float4*>(c.resid + (size_t)row * c.N + col) = x;
            *reinterpret_cast<uint2*>(c.out_bf16 + (size_t)row * c.ld_bf16 + col) =
                make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
        }
    }
    __syncwarp();  // the next block overwrites the staging buffer
}

static_assert((BN / 32) % 2 == 0, "the residual epilogue walks column blocks in pairs");

// AHEAD: column blocks whose global reads are in flight while a block is written (2: the next two,
// double-buffered; 1: the next one, half the registers)
template <int AHEAD = 2>
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
    const ResidCtx c = resid_ctx(p, t, tacc, rbase, lane, stg, part);
    float* const out_partials = p.out_partials;
    const int tok0 = p.tok0, n_tiles = p.n_tiles;
    float ss[8];
    if constexpr (AHEAD == 2) {
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
    } else {
        float4 ra[8], wa[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            ss[i] = 0.f;
            ra[i] = wa[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        resid_load(c, 0, ra, wa);
#pragma unroll 1
        for (int j = 0; j < BN / 32; ++j) {
            resid_block(c, j, ra, wa, ss);
            if (j + 1 < BN / 32) resid_load(c, j + 1, ra, wa);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float x = ss[i];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        const int row = t.row_begin + rbase + 4 * i + (lane >> 3);
        if ((lane & 7) == 0 && row < t.row_end) out_partials[(size_t)(tok0 + row) * n_tiles + t.n_blk] = x;
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
        // argument values used in the loops, read once (see ResidCtx)
        const int nq = p.nq, nkv = p.nkv;
        uint16_t* const q_out = p.q_out;
        uint16_t* const kv_pool = p.kv_pool;
        const float* const rope_cos = p.rope_cos;
        const float* const rope_sin = p.rope_sin;
        const bool any_rope = n0 / d < nq + nkv;
        float x2[32], cs[32], sn[32];
#pragma unroll 1
        for (int j = 0; j < half / 32; ++j) {
            if (ok && any_rope) {
                const float4* c4 = reinterpret_cast<const float4*>(rope_cos + (size_t)pos * half + 32 * j);
                const float4* s4 = reinterpret_cast<const float4*>(rope_sin + (size_t)pos * half + 32 * j);
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
                const int kind = head < nq ? 0 : (head < nq + nkv ? 1 : 2);
                const int g = kind == 1 ? head - nq : head - nq - nkv;
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
                    uint16_t* dst = q_out + ((size_t)tok * nq + head) * d;
                    store_bf16x32(dst + 32 * j, v);
                    store_bf16x32(dst + half + 32 * j, x2);
                } else {
                    store_kv_row32(kv_pool + page_base, kind - 1, g, nkv, d, slot, 32 * j, v);
                    store_kv_row32(kv_pool + page_base, kind - 1, g, nkv, d, slot, half + 32 * j, x2);
                }
            }
        }
    }
}


// One CTA's part of a GEMM launch. `smem`: the 1024-byte-aligned dynamic shared memory (kGemmSmemBytes
// - 1024 bytes are used); `tmem_base`: a TMEM allocation of TMEM_COLS columns that the caller owns.
// Warps 0..5 take the roles above; further warps only join the two block-wide barriers. Without a
// work counter (p.tile_ctr == nullptr), CTA `cta` of `ncta` takes units cta, cta + ncta, ... . The
// body starts and ends on a block-wide barrier and invalidates every mbarrier it initialised before
// it returns, so that the caller may reuse all of the shared memory.
template <int EPI, int RESID_AHEAD = 2>
__device__ __forceinline__ void gemm_body(const CUtensorMap* tmA, const CUtensorMap* tmB, const GemmArgs& p,
                                          uint8_t* smem, uint32_t tmem_base, int cta, int ncta) {
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

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 4); }
        mbar_init(drain, 1);
        for (int u = 0; u < 4; ++u) { mbar_init(&unit_full[u], 1); mbar_init(&unit_empty[u], 5); }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(tmA);
        tma_prefetch_desc(tmB);
    }
    __syncthreads();
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
            int next = p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : cta;
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
                    tma_load_2d_hint(sa, tmA, &full[stage], kb * BK, t.a_row, a_policy);
                    tma_load_2d(sb, tmB, &full[stage], kb * BK, t.b_row);  // B maps hold 128-row boxes
                    tma_load_2d(sb + B_BYTES / 2, tmB, &full[stage], kb * BK, t.b_row + BN / 2);
                    pending[stage] = (int)phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if (kb == kb0 + kb_per - 1 - (STAGES < kb_per ? STAGES : kb_per - 1))
                        next = p.tile_ctr ? atomicAdd(p.tile_ctr, 1) : unit + ncta;
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
    } else if (warp < kGemmThreads / 32) {
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
                    epilogue_resid<RESID_AHEAD>(p, t, tacc, quarter * 32, lane, stg, nullptr, ws);
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
                    epilogue_resid<RESID_AHEAD>(p, t, tacc, quarter * 32, lane, stg, ks == 2 ? ws : nullptr, nullptr);
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
    if (threadIdx.x == 0)
        for (int i = 0; i < kBodyBarriers; ++i) mbar_inval(full + i);
}

}  // namespace gemm_impl
}  // namespace nf
