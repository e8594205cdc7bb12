// The persistent device-scheduled layer kernel (see nf_mega.h): one launch per layer runs the layer's
// GEMMs (one-CTA tcgen05 bodies with their fused epilogues), decode attention, its split-KV merge and
// the prefill attention, in the plan's issue order, with device-side completion counters in place of
// streams and events.
//
// Every body keeps its own barriers and shared-memory layout: the kernel allocates TMEM once (512
// columns, the most any body uses) and each body initialises its mbarriers on entry and invalidates
// them on exit, so the same shared memory serves the next one. All tcgen05 work is single-CTA
// (cta_group::1): the GEMM runs on one-CTA 128 x 256 tiles here, not on the CTA pairs of the stream
// executor.
//
// Ordering between CTAs. A CTA that finishes an operation makes its global writes visible to the
// async proxy (fence.proxy.async.global), meets its other threads at a block barrier, and one thread
// adds 1 to the operation's counter with release semantics. A CTA about to start an operation waits,
// on one thread with acquire loads and a time limit, until the counter of every operation it depends
// on equals the CTA count of that operation's lane, meets its other threads at a block barrier, and
// every thread fences the async proxy again before any TMA or bulk copy reads what the others wrote.
// Every CTA is resident for the whole launch (one per SM, grid <= SMs), and the list is in issue
// order, so the earliest unfinished operation always has all its CTAs running or about to run: no
// wait can be on work that cannot start. A wait that runs out records NF_ERR_DEVICE_TIMEOUT; the CTA
// then skips the rest of its list (still counting itself finished, so that no other CTA waits on it).
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_decode_body.cuh"
#include "nf_gemm_body.cuh"
#include "nf_mega.h"
#include "nf_prefill_body.cuh"
#include "nf_ptx.cuh"

namespace nf {
namespace {

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Waits until *ctr >= target (bounded). Returns false after limit_ns.
__device__ __forceinline__ bool wait_count(const int* ctr, int target, int* status, uint64_t limit_ns) {
    if (ld_acquire(ctr) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(ctr) < target) {
        if (globaltimer_ns() - t0 > limit_ns) {
            set_status(status, NF_ERR_DEVICE_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

__device__ __forceinline__ int lane_ctas(int lane, int n_attn) {
    return lane == LANE_ATTN ? n_attn : lane == LANE_GEMM ? (int)gridDim.x - n_attn : (int)gridDim.x;
}

__device__ __forceinline__ int trace_kind(int kind) {
    return kind == MEGA_PREFILL ? NF_KERNEL_PREFILL_ATTN
                                : (kind == MEGA_DECODE || kind == MEGA_MERGE) ? NF_KERNEL_DECODE_ATTN : NF_KERNEL_GEMM;
}

// Each body is a separate (not inlined) function, so that its registers are allocated for it alone
// rather than for the union of all bodies.
// The residual epilogue keeps one column block of reads in flight instead of two: its arguments are
// read through a pointer here (not from the kernel's constant bank), which costs the registers the
// second buffer would take.
template <int EPI>
__device__ __noinline__ void run_gemm(const CUtensorMap* tmA, const CUtensorMap* tmB, const GemmArgs& g, uint8_t* smem,
                                      uint32_t tmem, int cta, int ncta) {
    gemm_impl::gemm_body<EPI, 1>(tmA, tmB, g, smem, tmem, cta, ncta);
}

template <int NQ>
__device__ __noinline__ void run_decode(const CUtensorMap* tmQ, const DecodeArgs& a, uint8_t* smem, uint32_t tmem,
                                        int cta, int ncta) {
    decode_impl::decode_body<NQ>(tmQ, a, smem, tmem, cta, ncta);
}

__device__ __noinline__ void run_prefill(const CUtensorMap* tmQ, const PrefillArgs& a, uint8_t* smem, uint32_t tmem,
                                         int cta, int ncta) {
    prefill_impl::prefill_body(tmQ, a, smem, tmem, cta, ncta);
}

template <int NQ>
__global__ void __launch_bounds__(kMegaThreads, 1) mega_layer_kernel(const __grid_constant__ MegaParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint32_t tmem_slot;
    __shared__ int s_stop;
    const int warp = threadIdx.x >> 5;
    if (warp == 1) {
        tmem_alloc(&tmem_slot, kMegaTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const bool attn_cta = (int)blockIdx.x < P.n_attn;
    bool stopped = false;

    for (int i = 0; i < P.n_ops; ++i) {
        const MegaOp& op = P.ops[i];
        int cta = (int)blockIdx.x, ncta = (int)gridDim.x;
        if (op.lane == LANE_ATTN) {
            if (!attn_cta) continue;
            ncta = P.n_attn;
        } else if (op.lane == LANE_GEMM) {
            if (attn_cta) continue;
            cta -= P.n_attn;
            ncta -= P.n_attn;
        }
        uint64_t t_start = 0;
        if (!stopped) {
            if (threadIdx.x == 0) {
                bool ok = true;
                for (int k = 0; k < kMegaMaxDeps && ok; ++k) {
                    const int d = op.dep[k];
                    if (d >= 0)
                        ok = wait_count(P.done + d, lane_ctas(P.ops[d].lane, P.n_attn), P.status,
                                        P.wait_limit_ns ? P.wait_limit_ns : NF_WAIT_LIMIT_NS);
                }
                if (ok && *reinterpret_cast<volatile int*>(P.status) == NF_ERR_DEVICE_TIMEOUT) ok = false;
                s_stop = ok ? 0 : 1;
                t_start = globaltimer_ns();
            }
            __syncthreads();
            stopped = s_stop != 0;
        }
        if (!stopped) {
            fence_proxy_async_global();
            tc_fence_after();
            switch (op.kind) {
                case MEGA_QKV:
                    run_gemm<EPI_QKV>(&op.tmA, &op.tmB, op.g, smem, tmem, cta, ncta);
                    break;
                case MEGA_RESID:
                    run_gemm<EPI_RESID>(&op.tmA, &op.tmB, op.g, smem, tmem, cta, ncta);
                    break;
                case MEGA_SWIGLU:
                    run_gemm<EPI_SWIGLU>(&op.tmA, &op.tmB, op.g, smem, tmem, cta, ncta);
                    break;
                case MEGA_DECODE:
                    run_decode<NQ>(&op.tmA, op.d, smem, tmem, cta, ncta);
                    break;
                case MEGA_MERGE: {
                    // one (request, group of 8 query heads) per warp
                    const DecodeArgs& a = op.d;
                    constexpr int NG = NQ / decode_impl::MERGE_HEADS;
                    constexpr int WPC = kMegaThreads / 32;
                    const int units = (a.req_end - a.req_begin) * NG;
                    for (int u = cta * WPC + warp; u < units; u += ncta * WPC)
                        decode_impl::merge_heads_warp<NQ>(a, a.req_begin + u / NG,
                                                          (u % NG) * decode_impl::MERGE_HEADS, threadIdx.x & 31);
                    break;
                }
                case MEGA_PREFILL:
                    run_prefill(&op.tmA, op.p, smem, tmem, cta, ncta);
                    break;
                default:
                    break;
            }
            fence_proxy_async_global();
            tc_fence_before();
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            __threadfence();
            red_release_add(P.done + i, 1);
            if (P.trace != nullptr && !stopped) {
                const int e = atomicAdd(P.trace_ctr, 1);
                if (e < P.trace_cap) {
                    P.trace[e].kernel = trace_kind(op.kind);
                    P.trace[e].smid = (int32_t)smid();
                    P.trace[e].t_start = t_start;
                    P.trace[e].t_end = globaltimer_ns();
                }
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kMegaTmemCols);
    }
}

template <int NQ>
cudaError_t launch_nq(const MegaParams& p, int grid, cudaStream_t stream) {
    static int configured = 0;  // 1: attributes set and one CTA per SM fits; -1: it does not
    const int smem = mega_smem_bytes(NQ);
    if (configured == 0) {
        cudaError_t e = cudaFuncSetAttribute(mega_layer_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        int blocks = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, mega_layer_kernel<NQ>, kMegaThreads, smem);
        if (e != cudaSuccess) return e;
        configured = blocks >= 1 ? 1 : -1;
    }
    if (configured < 0) return cudaErrorInvalidConfiguration;
    mega_layer_kernel<NQ><<<grid, kMegaThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

int mega_smem_bytes(int nq) {
    int s = kGemmSmemBytes;
    const int dec = nq == 64 ? (int)decode_impl::TcCfg<64>::SMEM : (int)decode_impl::TcCfg<32>::SMEM;
    if (dec > s) s = dec;
    if ((int)prefill_impl::SMEM > s) s = (int)prefill_impl::SMEM;
    return s;
}

cudaError_t launch_mega(const MegaParams& p, int nq, int grid, cudaStream_t stream) {
    if (grid <= 0 || p.n_ops <= 0) return cudaSuccess;
    if (grid > device_sm_count()) return cudaErrorInvalidValue;  // every CTA must be resident at once
    if (nq == 32) return launch_nq<32>(p, grid, stream);
    if (nq == 64) return launch_nq<64>(p, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace nf
