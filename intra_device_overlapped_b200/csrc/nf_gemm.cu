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

#include "nf_gemm_body.cuh"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

using namespace gemm_impl;

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5;
    uint64_t t_start = 0;
    if (threadIdx.x == 0) t_start = globaltimer_ns();
    if (warp == 1) {
        tmem_alloc(&tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    gemm_body<EPI>(&tmA, &tmB, p, smem, tmem_base, (int)blockIdx.x, (int)gridDim.x);
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
                    epilogue_resid<2>(p, t, tacc, quarter * 32, lane, stg, nullptr, ws);
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
                    epilogue_resid<2>(p, t, tacc, quarter * 32, lane, stg, ks == 2 ? ws : nullptr, nullptr);
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
