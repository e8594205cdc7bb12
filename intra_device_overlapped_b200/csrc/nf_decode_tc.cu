// Paged GQA decode attention on the 5th-generation tensor cores (head dim 128).
//
// Decode attention is the memory-bound operation NanoFlow overlaps with the GEMMs of
// another nano-batch (README "Introduction"; arXiv abstract). On sm_100a the warp-level
// mma.sync path runs at a small fraction of the tcgen05 rate, so an attention kernel
// confined to a few SMs would be limited by it; this kernel issues tcgen05.mma instead.
//
// Work item = (decode request r, KV head g), all of its ctx_len[r] + 1 keys. Keys stream
// in chunks of 128 (8 pages): a TMA producer warp loads the chunk's K and V pages of head g
// into a 3-stage ring (64 KB per stage, 128-byte swizzle, each 64-column half of K or V one
// 16 KB region so that 8-row groups sit 1024 bytes apart). One thread issues
//   S^T[128 keys x 16] = K Q^T      (A = K chunk, K-major; B = the G query rows of head g)
//   O^T[128 d x 16]   += V^T P^T    (A = V chunk read MN-major; B = P, K-major)
// with fp32 accumulators in TMEM (two S buffers and O^T: 48 of 64 allocated columns).
// Four softmax warps read S^T from TMEM (thread = key), keep a per-head running maximum
// that moves only when a score exceeds it by more than 2^8 (rescaling O^T in TMEM then),
// write P as bf16 into shared memory and hand it back to the MMA thread.
// Work is dealt to persistent CTAs in contiguous ranges of equal key-chunk counts.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

constexpr int NS = 3;                       // K/V chunk stages
constexpr int CHUNK_KEYS = 128;
constexpr uint32_t REGION = 16384;          // 128 rows x 128 B
constexpr uint32_t KV_STAGE = 4 * REGION;   // K halves, then V halves
constexpr uint32_t QP_BYTES = 4096;         // 16 rows x 256 B as two 2 KB regions
constexpr int MAX_ITEM_PAGES = 1024;        // page list of one request held in shared memory
constexpr uint32_t TMEM_COLS = 64;
constexpr int LOADERS = 4;                  // warps 6..9: K/V page loads (cp.async)
constexpr int THREADS = (6 + LOADERS) * 32; // warp 0 Q loads (TMA), warp 1 MMA + TMEM, warps 2..5 softmax
constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(128, 16);
constexpr uint32_t IDESC_PV = umma_idesc_bf16_f32_amn(128, 16);
constexpr float LAZY = 8.0f;

constexpr uint32_t OFF_Q = NS * KV_STAGE;
constexpr uint32_t OFF_P = OFF_Q + 2 * QP_BYTES;
constexpr uint32_t OFF_PAGES = OFF_P + 2 * QP_BYTES;
constexpr uint32_t OFF_RED = OFF_PAGES + MAX_ITEM_PAGES * 4;
constexpr uint32_t OFF_BAR = OFF_RED + 4 * 16 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 24 * 8 + 16 + 1024;

// Walks the CTA's items (r, g) whose first key-chunk index lies in [lo, hi).
struct ItemIter {
    int r, g, nkeys, nch;
    long long w;  // work_off[r]
    bool valid;
};

__device__ __forceinline__ void iter_load_req(ItemIter& it, const DecodeArgs& a) {
    it.nkeys = a.ctx_len[it.r] + 1;
    it.nch = (it.nkeys + CHUNK_KEYS - 1) / CHUNK_KEYS;
    it.w = a.item_off[it.r];
}

__device__ __forceinline__ void iter_init(ItemIter& it, const DecodeArgs& a, long long lo, long long hi) {
    int low = a.req_begin, high = a.req_end - 1;
    while (low < high) {  // last request whose work starts at or before lo
        const int mid = (low + high + 1) >> 1;
        if ((long long)a.item_off[mid] <= lo) low = mid; else high = mid - 1;
    }
    it.r = low;
    iter_load_req(it, a);
    const long long off = lo - it.w;
    it.g = off <= 0 ? 0 : (int)((off + it.nch - 1) / it.nch);
    if (it.g >= a.nkv) {
        it.r += 1;
        it.g = 0;
        if (it.r < a.req_end) iter_load_req(it, a);
    }
    it.valid = it.r < a.req_end && it.w + (long long)it.g * it.nch < hi;
}

__device__ __forceinline__ void iter_next(ItemIter& it, const DecodeArgs& a, long long hi) {
    if (++it.g == a.nkv) {
        it.g = 0;
        if (++it.r < a.req_end) iter_load_req(it, a);
    }
    it.valid = it.r < a.req_end && it.w + (long long)it.g * it.nch < hi;
}

__device__ __forceinline__ bool wait_bcast(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                           int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__global__ void __launch_bounds__(THREADS, 1)
    decode_attention_tc_kernel(const __grid_constant__ CUtensorMap tmKV, const __grid_constant__ CUtensorMap tmQ,
                               const __grid_constant__ DecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* red = reinterpret_cast<float*>(smem + OFF_RED);  // [4 warps][16]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* kv_full = bars;            // [NS]
    uint64_t* kv_empty = bars + NS;      // [NS]
    uint64_t* q_full = bars + 2 * NS;    // [2]
    uint64_t* q_empty = q_full + 2;      // [2]
    uint64_t* s_full = q_empty + 2;      // [2]
    uint64_t* s_free = s_full + 2;       // [2]
    uint64_t* p_full = s_free + 2;       // [2]
    uint64_t* pv_done = p_full + 2;      // [2]
    uint64_t* o_free = pv_done + 2;      // [1]
    uint64_t* drain = o_free + 1;        // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t t_start = 0;
    if (threadIdx.x == 0) {
        t_start = globaltimer_ns();
        for (int i = 0; i < NS; ++i) { mbar_init(&kv_full[i], LOADERS * 32); mbar_init(&kv_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1);
            mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 4);
            mbar_init(&p_full[i], 4); mbar_init(&pv_done[i], 1);
        }
        mbar_init(o_free, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmKV);
        tma_prefetch_desc(&tmQ);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
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
        // ---------------- Q loads: the 16 query rows starting at head g * G of request r (TMA)
        ItemIter it;
        iter_init(it, a, lo, hi);
        uint32_t ni = 0;
        for (; it.valid; iter_next(it, a, hi), ++ni) {
            const uint32_t qb = ni & 1u;
            if (!wait_bcast(&q_empty[qb], ((ni >> 1) & 1u) ^ 1u, abort_flag, a.status, lane)) break;
            if (lane == 0) {
                uint8_t* qd = smem + OFF_Q + qb * QP_BYTES;
                mbar_arrive_expect_tx(&q_full[qb], QP_BYTES);
                const int y = it.r * a.nq + it.g * a.G;
                tma_load_2d(qd, &tmQ, &q_full[qb], 0, y);
                tma_load_2d(qd + 2048, &tmQ, &q_full[qb], 64, y);
            }
        }
        if (lane == 0) {  // the last Q copy must land before the CTA exits
            volatile int quiet = 0;
            if (ni > 0) mbar_wait(&q_full[(ni - 1) & 1u], ((ni - 1) >> 1) & 1u, &quiet, nullptr);
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ---------------- K/V loader warps: each chunk is 8 pages x (K, V) blocks of 4 KB
        // (16 keys x 256 B, contiguous in the pool); consecutive threads copy consecutive 16 B
        // of a block into its 128-byte-swizzled place. Keys past the request are zero-filled.
        // Each loader thread arrives (no-increment) on the stage barrier when its copies land.
        const int t = threadIdx.x - 6 * 32;              // 0 .. 127
        ItemIter it;
        iter_init(it, a, lo, hi);
        uint32_t cs = 0;
        bool ok = true;
        const char* pool = reinterpret_cast<const char*>(a.kv_pool);
        for (; it.valid && ok; iter_next(it, a, hi)) {
            const int npages = (it.nkeys + 15) >> 4;
            const int base = a.page_indptr[it.r];
            for (int c = 0; c < it.nch && ok; ++c, ++cs) {
                const int st = (int)(cs % NS);
                if (!wait_bcast(&kv_empty[st], ((cs / NS) & 1u) ^ 1u, abort_flag, a.status, lane)) { ok = false; break; }
                const uint32_t sdst = sbase + st * KV_STAGE;
                const int np = min(8, npages - 8 * c);
                // this thread's page ids for the chunk: block index (i*128 + t) >> 8 = 2 j + isv
                int pgs[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    int pg = 0;
                    if (j < np) {
                        pg = __ldg(a.page_indices + base + 8 * c + j);
                        if (pg < 0 || pg >= a.num_pages) { set_status(a.status, NF_ERR_DEVICE_BOUNDS); pg = 0; }
                    }
                    pgs[j] = pg;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    // 16-byte chunk i * 128 + t of the stage: block (i >> 1) = 2 j + isv, chunk b in the block
                    const int j = i >> 2, isv = (i >> 1) & 1;
                    const int b = (i & 1) * 128 + t;
                    const int kr = b >> 4, cc = b & 15;
                    const bool valid = j < np && (8 * c + j) * 16 + kr < it.nkeys;
                    const char* src = pool + ((((size_t)pgs[j] * 2 + isv) * a.nkv + it.g) * 16 + kr) * 256 + cc * 16;
                    const uint32_t dst = sdst + isv * 2 * REGION + (cc >> 3) * REGION + j * 2048 + kr * 128 +
                                         ((((cc & 7) ^ (kr & 7))) << 4);
                    cp_async_16(dst, valid ? (const void*)src : (const void*)pool, valid ? 16u : 0u);
                }
                cp_async_arrive_noinc(&kv_full[st]);
            }
        }
        // let this thread's copies land before the CTA exits
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            ItemIter it;
            iter_init(it, a, lo, hi);
            uint32_t cs = 0, ni = 0;
            bool ok = true;
            auto issue_pv = [&](uint32_t x, bool first) -> bool {
                const uint32_t pb = x & 1u;
                if (!mbar_wait(&p_full[pb], (x >> 1) & 1u, abort_flag, a.status)) return false;
                if (first && !mbar_wait(o_free, (ni & 1u) ^ 1u, abort_flag, a.status)) return false;
                tc_fence_after();
                const uint32_t st = x % NS;
                const uint32_t vbase = sbase + st * KV_STAGE + 2 * REGION;
                const uint32_t pbase = sbase + OFF_P + pb * QP_BYTES;
#pragma unroll
                for (int kk = 0; kk < CHUNK_KEYS / 16; ++kk) {
                    const uint64_t ad = umma_desc_sw128_mn(vbase + kk * 2048, REGION, 1024);
                    const uint64_t bd = umma_desc_sw128(pbase + (kk >> 2) * 2048 + (kk & 3) * 32);
                    umma_bf16(tmem + 32, ad, bd, IDESC_PV, (first && kk == 0) ? 0u : 1u);
                }
                umma_commit(&pv_done[pb]);
                umma_commit(&kv_empty[st]);
                return true;
            };
            for (; it.valid && ok; iter_next(it, a, hi), ++ni) {
                const uint32_t qb = ni & 1u;
                if (!mbar_wait(&q_full[qb], (ni >> 1) & 1u, abort_flag, a.status)) { ok = false; break; }
                const uint32_t qbase = sbase + OFF_Q + qb * QP_BYTES;
                for (int c = 0; c < it.nch; ++c, ++cs) {
                    const uint32_t st = cs % NS, sb = cs & 1u;
                    if (!mbar_wait(&kv_full[st], (cs / NS) & 1u, abort_flag, a.status)) { ok = false; break; }
                    if (!mbar_wait(&s_free[sb], ((cs >> 1) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
                    fence_proxy_async_smem();  // cp.async data -> tensor-core reads
                    tc_fence_after();
                    const uint32_t kbase = sbase + st * KV_STAGE;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t ad = umma_desc_sw128(kbase + (kk >> 2) * REGION + (kk & 3) * 32);
                        const uint64_t bd = umma_desc_sw128(qbase + (kk >> 2) * 2048 + (kk & 3) * 32);
                        umma_bf16(tmem + sb * 16, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[sb]);
                    if (c == it.nch - 1) umma_commit(&q_empty[qb]);
                    if (c > 0 && !issue_pv(cs - 1, c == 1)) { ok = false; break; }
                }
                if (!ok) break;
                if (!issue_pv(cs - 1, it.nch == 1)) { ok = false; break; }
            }
            umma_commit(drain);
            volatile int quiet = 0;
            mbar_wait(drain, 0, &quiet, nullptr);
        }
        __syncwarp();
    } else {
        // ---------------- softmax warps: thread = one key of the chunk (TMEM lane)
        // Control flow is uniform across the four warps (every named barrier is reached by all
        // 128 threads); a failed wait is carried in `okc` and all warps leave together.
        const int q = warp & 3;
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        ItemIter it;
        iter_init(it, a, lo, hi);
        uint32_t cs = 0, ni = 0;
        bool ok = true;
        for (; it.valid && ok; iter_next(it, a, hi), ++ni) {
            float m[8], lp[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) { m[h] = -INFINITY; lp[h] = 0.f; }
            for (int c = 0; c < it.nch; ++c, ++cs) {
                const uint32_t sb = cs & 1u;
                bool okc = wait_bcast(&s_full[sb], (cs >> 1) & 1u, abort_flag, a.status, lane);
                float s[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) s[h] = -INFINITY;
                if (okc) {
                    tc_fence_after();
                    tmem_ld16(tmem + lane_addr + sb * 16, s);
                    tc_fence_before();
                }
                __syncwarp();
                if (lane == 0 && okc) mbar_arrive(&s_free[sb]);
                const int jl = q * 32 + lane;               // key within the chunk
                const bool valid = okc && c * CHUNK_KEYS + jl < it.nkeys;
                bool need = false;
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    s[h] = (valid && h < a.G) ? s[h] * a.scale_log2 : -INFINITY;
                    need |= s[h] > m[h] + LAZY;
                }
                if (bar_red_or(1, 128, need)) {
                    // exact new maximum per head over the chunk's 128 keys
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        float x = s[h];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                        if (lane == 0) red[q * 16 + h] = x;
                    }
                    bar_sync_n(2, 128);
                    float cf[8];
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const float x = fmaxf(fmaxf(red[h], red[16 + h]), fmaxf(red[32 + h], red[48 + h]));
                        const float nm = fmaxf(m[h], x);
                        cf[h] = (nm == -INFINITY) ? 1.f : exp2f(m[h] - nm);
                        m[h] = nm;
                        lp[h] *= cf[h];
                    }
                    if (c > 0) {
                        // the previous chunk's P V must have landed in O^T before it is rescaled
                        okc = okc && wait_bcast(&pv_done[(cs - 1) & 1u], ((cs - 1) >> 1) & 1u, abort_flag, a.status,
                                                lane);
                        if (okc) {
                            tc_fence_after();
                            float o[16];
                            tmem_ld16(tmem + lane_addr + 32, o);
#pragma unroll
                            for (int h = 0; h < 8; ++h) o[h] *= cf[h];
                            tmem_st16(tmem + lane_addr + 32, o);
                            tc_fence_before();
                        }
                    }
                    bar_sync_n(2, 128);
                }
                // P (bf16) of this thread's key for each head, into the P buffer of this chunk
                const uint32_t pb = cs & 1u;
                if (cs >= 2) okc = okc && wait_bcast(&pv_done[pb], ((cs - 2) >> 1) & 1u, abort_flag, a.status, lane);
                if (okc) {
                    uint8_t* pbuf = smem + OFF_P + pb * QP_BYTES + (jl >> 6) * 2048;
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        if (h < a.G) {
                            const float p = exp2f(s[h] - m[h]);  // 0 for masked keys
                            lp[h] += p;
                            *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128_offset(h, jl & 63)) = __float2bfloat16_rn(p);
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && okc) mbar_arrive(&p_full[pb]);
                if (bar_red_or(3, 128, !okc)) { ok = false; break; }
            }
            if (!ok) break;
            // ---- item output: O^T (thread = one d) / l per head
            bool okc = wait_bcast(&pv_done[(cs - 1) & 1u], ((cs - 1) >> 1) & 1u, abort_flag, a.status, lane);
            float o[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) o[h] = 0.f;
            if (okc) {
                tc_fence_after();
                tmem_ld16(tmem + lane_addr + 32, o);
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0 && okc) mbar_arrive(o_free);
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                float x = lp[h];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
                if (lane == 0) red[q * 16 + h] = x;
            }
            bar_sync_n(2, 128);
            if (okc) {
                const int d = q * 32 + lane;
                uint16_t* ob = a.out + ((size_t)it.r * a.nq + (size_t)it.g * a.G) * 128 + d;
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    if (h < a.G) {
                        const float l = red[h] + red[16 + h] + red[32 + h] + red[48 + h];
                        ob[(size_t)h * 128] = f2bf(o[h] / l);
                    }
                }
            }
            if (bar_red_or(2, 128, !okc)) { ok = false; break; }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
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

}  // namespace

int decode_tc_smem_bytes() { return (int)SMEM_BYTES; }

cudaError_t launch_decode_attention_tc(const CUtensorMap& tmKV, const CUtensorMap& tmQ, const DecodeArgs& a,
                                       int grid, cudaStream_t stream) {
    if (grid <= 0 || a.req_end <= a.req_begin) return cudaSuccess;
    static bool cfg = false;
    if (!cfg) {
        cudaError_t e = cudaFuncSetAttribute(decode_attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        cfg = true;
    }
    decode_attention_tc_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(tmKV, tmQ, a);
    return cudaGetLastError();
}

}  // namespace nf
