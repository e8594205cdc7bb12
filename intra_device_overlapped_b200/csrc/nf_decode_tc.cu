// Paged GQA decode attention on the 5th-generation tensor cores (8 KV heads of dim 128).
//
// Decode attention is the memory-bound operation NanoFlow overlaps with the GEMMs of
// another nano-batch (README "Introduction"; arXiv abstract). For the overlap to pay, the
// attention kernel must pull HBM bandwidth from a minority of the SMs, and on B200 one SM's
// DRAM throughput grows with the size of each transfer (about 45 GB/s per SM with 2 KB
// transfers, about 190 GB/s with 64 KB ones). The paged KV cache is therefore laid out so
// that one page of one layer -- K and V of all KV heads, 64 KB -- is a single contiguous
// block whose bytes are already the shared-memory image the tensor cores read:
//   [K|V][64-column half of d][KV head][16 tokens][8 chunks of 16 B, chunk c of row r at c ^ (r & 7)]
// and one bulk copy moves a whole page into a ring stage.
//
// Work item = one decode request with all of its heads; a stage is one page (16 keys x 8
// KV heads = 128 rows). One thread issues
//   S^T[128 rows x nq] = K_page Q^T       (A = K, K-major; B = the request's nq query rows)
//   O^T[128 d x nq]   += V_page^T P^T     (A = V read MN-major; B = P, K-major)
// with fp32 accumulators in TMEM. A row (KV head h, key k) of S^T only pairs with the G query
// heads of head h, so P is block diagonal: each softmax thread owns one row, writes its G
// probabilities and leaves the other entries at the zero they were set to once. Per query
// head the running maximum moves only when a score exceeds it by more than 2^8 (O^T is then
// rescaled in TMEM). Requests are dealt to persistent CTAs in contiguous ranges of equal
// page counts; there is no split-KV merge.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

constexpr int ROWS = 128;                   // 8 KV heads x 16 keys of one page
constexpr uint32_t PAGE_BYTES = 65536;      // K and V of all heads of one page
constexpr uint32_t REGION = 16384;          // one 64-column half of K or V: 128 rows x 128 B
constexpr float LAZY = 8.0f;

template <int NQ>
struct TcCfg {
    static constexpr int NS = NQ <= 32 ? 3 : 2;           // page stages
    static constexpr uint32_t QB = NQ * 256;              // Q: two halves of NQ rows x 128 B
    static constexpr uint32_t PB = NQ * 256;              // P buffer: two key halves of NQ rows x 128 B
    static constexpr uint32_t OFF_Q = NS * PAGE_BYTES;
    static constexpr uint32_t OFF_P = OFF_Q + QB;
    static constexpr uint32_t OFF_CF = OFF_P + 2 * PB;    // float[NQ] rescale factors / row sums
    static constexpr uint32_t OFF_BAR = OFF_CF + NQ * 4;
    static constexpr uint32_t SMEM = OFF_BAR + 32 * 8 + 1024;
    static constexpr uint32_t TMEM_COLS = NQ <= 32 ? 128 : 256;  // S[2] + O^T: 3 NQ columns
    static constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(128, NQ);
    static constexpr uint32_t IDESC_PV = umma_idesc_bf16_f32_amn(128, NQ);
};

constexpr int THREADS = 192;  // warp 0 loads (Q by TMA, pages by bulk copy), warp 1 MMA + TMEM, warps 2..5 softmax

// Walks the CTA's requests whose first page index (in the page-prefix work space) is in [lo, hi).
struct ReqIter {
    int r, nkeys, npages;
    long long w;
    bool valid;
};

__device__ __forceinline__ void req_load(ReqIter& it, const DecodeArgs& a) {
    it.nkeys = a.ctx_len[it.r] + 1;
    it.npages = (it.nkeys + 15) >> 4;
    it.w = a.item_off[it.r];
}

__device__ __forceinline__ void req_init(ReqIter& it, const DecodeArgs& a, long long lo, long long hi) {
    int low = a.req_begin, high = a.req_end - 1;
    while (low < high) {  // last request whose work starts at or before lo
        const int mid = (low + high + 1) >> 1;
        if ((long long)a.item_off[mid] <= lo) low = mid; else high = mid - 1;
    }
    it.r = low;
    req_load(it, a);
    if (it.w < lo) {  // starts before lo: belongs to the previous CTA
        it.r += 1;
        if (it.r < a.req_end) req_load(it, a);
    }
    it.valid = it.r < a.req_end && it.w < hi;
}

__device__ __forceinline__ void req_next(ReqIter& it, const DecodeArgs& a, long long hi) {
    if (++it.r < a.req_end) req_load(it, a);
    it.valid = it.r < a.req_end && it.w < hi;
}

__device__ __forceinline__ bool wait_bcast(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                           int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <int NQ>
__global__ void __launch_bounds__(THREADS, 1)
    decode_attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ DecodeArgs a) {
    using C = TcCfg<NQ>;
    constexpr int NS = C::NS;
    constexpr int G = NQ / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* cfs = reinterpret_cast<float*>(smem + C::OFF_CF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* kv_full = bars;            // [NS]
    uint64_t* kv_empty = bars + NS;      // [NS]
    uint64_t* q_full = bars + 2 * NS;    // [1]
    uint64_t* q_empty = q_full + 1;      // [1]
    uint64_t* s_full = q_empty + 1;      // [2]
    uint64_t* s_free = s_full + 2;       // [2]
    uint64_t* p_full = s_free + 2;       // [2]
    uint64_t* pv_done = p_full + 2;      // [2]
    uint64_t* o_free = pv_done + 2;      // [1]
    uint64_t* drain = o_free + 1;        // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t t_start = 0;
    // P buffers start at zero: only the block-diagonal entries are ever written
    for (uint32_t i = threadIdx.x; i < 2 * C::PB / 16; i += THREADS)
        reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) {
        t_start = globaltimer_ns();
        for (int i = 0; i < NS; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 4);
            mbar_init(&p_full[i], 4); mbar_init(&pv_done[i], 1);
        }
        mbar_init(o_free, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    fence_proxy_async_smem();  // zeroed P buffers -> tensor-core reads
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sbase = smem_u32(smem);

    const long long W0 = a.item_off[a.req_begin];
    const long long W = (long long)a.item_off[a.req_end] - W0;
    const long long lo = W0 + W * blockIdx.x / gridDim.x;
    const long long hi = W0 + W * (blockIdx.x + 1) / gridDim.x;

    if (warp == 0) {
        // ---------------- loader warp: Q of the request (TMA, two 64-column halves of NQ rows),
        // then each page with one 64 KB bulk copy. Page ids are read 32 at a time (one per lane)
        // and handed to lane 0 with shuffles.
        ReqIter it;
        req_init(it, a, lo, hi);
        uint32_t cs = 0, ni = 0;
        bool ok = true;
        const char* pool = reinterpret_cast<const char*>(a.kv_pool);
        for (; it.valid && ok; req_next(it, a, hi), ++ni) {
            const int base = a.page_indptr[it.r];
            if (!wait_bcast(q_empty, (ni & 1u) ^ 1u, abort_flag, a.status, lane)) { ok = false; break; }
            if (lane == 0) {
                uint8_t* qd = smem + C::OFF_Q;
                mbar_arrive_expect_tx(q_full, C::QB);
                tma_load_2d(qd, &tmQ, q_full, 0, it.r * NQ);
                tma_load_2d(qd + NQ * 128, &tmQ, q_full, 64, it.r * NQ);
            }
            int ids = 0;
            for (int j = 0; j < it.npages; ++j, ++cs) {
                if ((j & 31) == 0) {
                    const int jj = j + lane;
                    ids = jj < it.npages ? __ldg(a.page_indices + base + jj) : 0;
                    if (ids < 0 || ids >= a.num_pages) { set_status(a.status, NF_ERR_DEVICE_BOUNDS); ids = 0; }
                }
                const int pg = __shfl_sync(0xffffffffu, ids, j & 31);
                const int st = (int)(cs % NS);
                if (!wait_bcast(&kv_empty[st], ((cs / NS) & 1u) ^ 1u, abort_flag, a.status, lane)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&kv_full[st], PAGE_BYTES);
                    bulk_load(smem + st * PAGE_BYTES, pool + (size_t)pg * PAGE_BYTES, PAGE_BYTES, &kv_full[st]);
                }
            }
        }
        if (lane == 0) {
            // let the copies still in flight land before the CTA exits
            volatile int quiet = 0;
            for (uint32_t x = cs > (uint32_t)NS ? cs - NS : 0u; x < cs; ++x)
                mbar_wait(&kv_full[x % NS], (x / NS) & 1u, &quiet, nullptr);
            if (ni > 0) mbar_wait(q_full, (ni - 1) & 1u, &quiet, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            ReqIter it;
            req_init(it, a, lo, hi);
            uint32_t cs = 0, ni = 0;
            bool ok = true;
            const uint32_t qbase = sbase + C::OFF_Q;
            auto issue_pv = [&](uint32_t x, bool first) -> bool {
                const uint32_t pb = x & 1u;
                if (!mbar_wait(&p_full[pb], (x >> 1) & 1u, abort_flag, a.status)) return false;
                if (first && !mbar_wait(o_free, (ni & 1u) ^ 1u, abort_flag, a.status)) return false;
                tc_fence_after();
                const uint32_t vbase = sbase + (x % NS) * PAGE_BYTES + 2 * REGION;
                const uint32_t pbase = sbase + C::OFF_P + pb * C::PB;
#pragma unroll
                for (int kk = 0; kk < ROWS / 16; ++kk) {
                    const uint64_t ad = umma_desc_sw128_mn(vbase + kk * 2048, REGION, 1024);
                    const uint64_t bd = umma_desc_sw128(pbase + (kk >> 2) * (NQ * 128) + (kk & 3) * 32);
                    umma_bf16(tmem + 2 * NQ, ad, bd, C::IDESC_PV, (first && kk == 0) ? 0u : 1u);
                }
                umma_commit(&pv_done[pb]);
                umma_commit(&kv_empty[x % NS]);
                return true;
            };
            for (; it.valid && ok; req_next(it, a, hi), ++ni) {
                if (!mbar_wait(q_full, ni & 1u, abort_flag, a.status)) { ok = false; break; }
                for (int c = 0; c < it.npages; ++c, ++cs) {
                    const uint32_t st = cs % NS, sb = cs & 1u;
                    if (!mbar_wait(&kv_full[st], (cs / NS) & 1u, abort_flag, a.status)) { ok = false; break; }
                    if (!mbar_wait(&s_free[sb], ((cs >> 1) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t kbase = sbase + st * PAGE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t ad = umma_desc_sw128(kbase + (kk >> 2) * REGION + (kk & 3) * 32);
                        const uint64_t bd = umma_desc_sw128(qbase + (kk >> 2) * (NQ * 128) + (kk & 3) * 32);
                        umma_bf16(tmem + sb * NQ, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[sb]);
                    if (c == it.npages - 1) umma_commit(q_empty);
                    if (c > 0 && !issue_pv(cs - 1, c == 1)) { ok = false; break; }
                }
                if (!ok) break;
                if (!issue_pv(cs - 1, it.npages == 1)) { ok = false; break; }
            }
            umma_commit(drain);
            volatile int quiet = 0;
            mbar_wait(drain, 0, &quiet, nullptr);
        }
        __syncwarp();
    } else {
        // ---------------- softmax warps: thread = row (KV head h = t / 16, key k = t % 16) of the page.
        // Every named barrier is reached by all 128 threads; failed waits travel in `okc`.
        const int q = warp & 3;
        const int t = q * 32 + lane;          // row
        const int h = t >> 4, k = t & 15;
        const int hsel = lane >> 4;           // which of the warp's two heads this lane's row belongs to
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        ReqIter it;
        req_init(it, a, lo, hi);
        uint32_t cs = 0, ni = 0;
        bool ok = true;
        for (; it.valid && ok; req_next(it, a, hi), ++ni) {
            float m[G], lp[G];
#pragma unroll
            for (int i = 0; i < G; ++i) { m[i] = -INFINITY; lp[i] = 0.f; }
            for (int c = 0; c < it.npages; ++c, ++cs) {
                const uint32_t sb = cs & 1u;
                bool okc = wait_bcast(&s_full[sb], (cs >> 1) & 1u, abort_flag, a.status, lane);
                float sw[2 * G];  // scores of the warp's two heads' query columns
#pragma unroll
                for (int i = 0; i < 2 * G; ++i) sw[i] = -INFINITY;
                if (okc) {
                    tc_fence_after();
                    float tmp[16];
                    tmem_ld16(tmem + lane_addr + sb * NQ + ((2 * q * G) & ~15), tmp);
                    const int off = (2 * q * G) & 15;
#pragma unroll
                    for (int i = 0; i < 2 * G; ++i) sw[i] = tmp[(off + i) & 15];
                    tc_fence_before();
                }
                __syncwarp();
                if (lane == 0 && okc) mbar_arrive(&s_free[sb]);
                const bool valid = okc && c * 16 + k < it.nkeys;
                float s[G];
                bool need = false;
#pragma unroll
                for (int i = 0; i < G; ++i) {
                    const float x = hsel ? sw[G + i] : sw[i];
                    s[i] = valid ? x * a.scale_log2 : -INFINITY;
                    need |= s[i] > m[i] + LAZY;
                }
                if (bar_red_or(1, 128, need)) {
                    // exact page maximum per query head over the head's 16 keys (one half-warp)
                    float cf[G];
#pragma unroll
                    for (int i = 0; i < G; ++i) {
                        float x = s[i];
#pragma unroll
                        for (int o = 8; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                        const float nm = fmaxf(m[i], x);
                        cf[i] = (nm == -INFINITY) ? 1.f : exp2f(m[i] - nm);
                        m[i] = nm;
                        lp[i] *= cf[i];
                    }
                    if (c > 0) {
                        if (k == 0) {
#pragma unroll
                            for (int i = 0; i < G; ++i) cfs[h * G + i] = cf[i];
                        }
                        bar_sync_n(2, 128);
                        // the previous page's P V must have landed in O^T before it is rescaled
                        okc = okc && wait_bcast(&pv_done[(cs - 1) & 1u], ((cs - 1) >> 1) & 1u, abort_flag,
                                                a.status, lane);
                        if (okc) {
                            tc_fence_after();
#pragma unroll
                            for (int c16 = 0; c16 < NQ / 16; ++c16) {
                                float o[16];
                                tmem_ld16(tmem + lane_addr + 2 * NQ + c16 * 16, o);
#pragma unroll
                                for (int i = 0; i < 16; ++i) o[i] *= cfs[c16 * 16 + i];
                                tmem_st16(tmem + lane_addr + 2 * NQ + c16 * 16, o);
                            }
                            tc_fence_before();
                        }
                        bar_sync_n(2, 128);
                    }
                }
                // P entries of this row (its G query heads) into this page's P buffer
                const uint32_t pb = cs & 1u;
                if (cs >= 2) okc = okc && wait_bcast(&pv_done[pb], ((cs - 2) >> 1) & 1u, abort_flag, a.status, lane);
                if (okc) {
                    uint8_t* pbuf = smem + C::OFF_P + pb * C::PB + (t >> 6) * (NQ * 128);
#pragma unroll
                    for (int i = 0; i < G; ++i) {
                        const float p = exp2f(s[i] - m[i]);  // 0 for masked keys
                        lp[i] += p;
                        *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128_offset(h * G + i, t & 63)) =
                            __float2bfloat16_rn(p);
                    }
                    if (c * 16 + k >= it.nkeys) {
                        // V row of a key past the request: zero it so that 0 * garbage cannot occur
                        uint8_t* vrow = smem + (cs % NS) * PAGE_BYTES + 2 * REGION + t * 128;
#pragma unroll
                        for (int b = 0; b < 2; ++b)
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                reinterpret_cast<uint4*>(vrow + b * REGION)[i] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && okc) mbar_arrive(&p_full[pb]);
                if (bar_red_or(3, 128, !okc)) { ok = false; break; }
            }
            if (!ok) break;
            // ---- request output: O^T (thread = one d) / l per query head
#pragma unroll
            for (int i = 0; i < G; ++i) {
                float x = lp[i];
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (k == 0) cfs[h * G + i] = x;
            }
            bool okc = wait_bcast(&pv_done[(cs - 1) & 1u], ((cs - 1) >> 1) & 1u, abort_flag, a.status, lane);
            bar_sync_n(2, 128);
            uint16_t* ob = a.out + (size_t)it.r * NQ * 128 + t;  // thread t writes d = t of every head
            if (okc) tc_fence_after();
#pragma unroll
            for (int c16 = 0; c16 < NQ / 16; ++c16) {
                float o[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] = 0.f;
                if (okc) {
                    tmem_ld16(tmem + lane_addr + 2 * NQ + c16 * 16, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i) ob[(size_t)(c16 * 16 + i) * 128] = f2bf(o[i] / cfs[c16 * 16 + i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && okc) mbar_arrive(o_free);
            if (bar_red_or(2, 128, !okc)) { ok = false; break; }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (threadIdx.x == 0 && a.trace != nullptr) {
        const int i = atomicAdd(a.trace_ctr, 1);
        if (i < a.trace_cap) {
            a.trace[i].kernel = NF_KERNEL_DECODE_ATTN;
            a.trace[i].smid = (int32_t)smid();
            a.trace[i].t_start = t_start;
            a.trace[i].t_end = globaltimer_ns();
        }
    }
}

template <int NQ>
cudaError_t launch_nq(const CUtensorMap& tmQ, const DecodeArgs& a, int grid, cudaStream_t stream) {
    static bool cfg = false;
    if (!cfg) {
        cudaError_t e = cudaFuncSetAttribute(decode_attention_tc_kernel<NQ>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TcCfg<NQ>::SMEM);
        if (e != cudaSuccess) return e;
        cfg = true;
    }
    decode_attention_tc_kernel<NQ><<<grid, THREADS, TcCfg<NQ>::SMEM, stream>>>(tmQ, a);
    return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(int nq, int nkv, int head_dim) {
    return head_dim == 128 && nkv == 8 && (nq == 32 || nq == 64);
}

cudaError_t launch_decode_attention_tc(const CUtensorMap& tmQ, const DecodeArgs& a, int grid, cudaStream_t stream) {
    if (grid <= 0 || a.req_end <= a.req_begin) return cudaSuccess;
    if (a.nq == 32) return launch_nq<32>(tmQ, a, grid, stream);
    if (a.nq == 64) return launch_nq<64>(tmQ, a, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace nf
