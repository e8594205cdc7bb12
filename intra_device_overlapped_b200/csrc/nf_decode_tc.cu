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
constexpr int PREFETCH_CHUNKS = 4;          // L2 bulk prefetch runs this many chunks ahead of the TMA loads
constexpr uint32_t TMEM_COLS = 64;
constexpr int THREADS = 192;                // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 softmax
constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(128, 16);
constexpr uint32_t IDESC_PV = umma_idesc_bf16_f32_amn(128, 16);
constexpr float LAZY = 8.0f;

constexpr uint32_t OFF_Q = NS * KV_STAGE;
constexpr uint32_t OFF_P = OFF_Q + 2 * QP_BYTES;
constexpr uint32_t OFF_PAGES = OFF_P + 2 * QP_BYTES;
constexpr uint32_t OFF_RED = OFF_PAGES + 2 * MAX_ITEM_PAGES * 4;
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
    int* pages_sm = reinterpret_cast<int*>(smem + OFF_PAGES);
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
        for (int i = 0; i < NS; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
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
        // ---------------- TMA producer. Two cursors walk the CTA's chunk sequence: the
        // prefetch cursor (page lists staged in shared memory, K and V page blocks prefetched
        // into L2) runs PREFETCH_CHUNKS ahead of the TMA cursor (loads into the ring), and at
        // most one item ahead, so item k's page list sits in buffer k & 1 for both.
        ItemIter tit, pit;
        iter_init(tit, a, lo, hi);
        pit = tit;
        uint32_t cs = 0, tni = 0, tc = 0;     // TMA cursor: chunk seq, item seq, chunk in item
        uint32_t pcs = 0, pni = 0, pc = 0;    // prefetch cursor
        bool ok = true;
        const size_t blk = (size_t)16 * 128;  // elements of one page block of one KV head
        auto stage_list = [&](const ItemIter& x, uint32_t seq) {
            int* buf = pages_sm + (seq & 1u) * MAX_ITEM_PAGES;
            const int npages = (x.nkeys + 15) >> 4;
            const int base = a.page_indptr[x.r];
            for (int j = lane; j < npages && j < MAX_ITEM_PAGES; j += 32) {
                int pg = a.page_indices[base + j];
                if (pg < 0 || pg >= a.num_pages) { set_status(a.status, NF_ERR_DEVICE_BOUNDS); pg = 0; }
                buf[j] = pg;
            }
            __syncwarp();
        };
        if (pit.valid) stage_list(pit, 0);
        while (tit.valid && ok) {
            // ---- prefetch cursor: keep PREFETCH_CHUNKS chunks ahead
            while (pit.valid && pcs < cs + PREFETCH_CHUNKS) {
                if (pc == (uint32_t)pit.nch) {          // this item is prefetched: move to the next one
                    if (pni > tni) break;               // never two items ahead of the TMA cursor
                    iter_next(pit, a, hi);
                    ++pni;
                    pc = 0;
                    if (!pit.valid) break;
                    stage_list(pit, pni);
                    continue;
                }
                const int* buf = pages_sm + (pni & 1u) * MAX_ITEM_PAGES;
                const int npages = (pit.nkeys + 15) >> 4;
                const int j0 = 8 * (int)pc, np = min(8, npages - j0);
                if (lane < 2 * np) {
                    const int pg = buf[min(j0 + (lane >> 1), MAX_ITEM_PAGES - 1)];
                    const uint16_t* src = a.kv_pool + (((size_t)pg * 2 + (lane & 1)) * a.nkv + pit.g) * blk;
                    prefetch_l2_bulk(src, (uint32_t)(blk * 2));
                }
                ++pcs;
                ++pc;
            }
            // ---- TMA cursor: one chunk into the ring
            if (tc == 0) {
                const uint32_t qb = tni & 1u;
                if (!wait_bcast(&q_empty[qb], ((tni >> 1) & 1u) ^ 1u, abort_flag, a.status, lane)) { ok = false; break; }
                if (lane == 0) {
                    uint8_t* qd = smem + OFF_Q + qb * QP_BYTES;
                    mbar_arrive_expect_tx(&q_full[qb], QP_BYTES);
                    const int y = tit.r * a.nq + tit.g * a.G;
                    tma_load_2d(qd, &tmQ, &q_full[qb], 0, y);
                    tma_load_2d(qd + 2048, &tmQ, &q_full[qb], 64, y);
                }
            }
            const int st = (int)(cs % NS);
            if (!wait_bcast(&kv_empty[st], ((cs / NS) & 1u) ^ 1u, abort_flag, a.status, lane)) { ok = false; break; }
            if (lane == 0) {
                const int* buf = pages_sm + (tni & 1u) * MAX_ITEM_PAGES;
                const int npages = (tit.nkeys + 15) >> 4;
                const int np = min(8, npages - 8 * (int)tc);
                uint8_t* kd = smem + st * KV_STAGE;
                uint8_t* vd = kd + 2 * REGION;
                mbar_arrive_expect_tx(&kv_full[st], (uint32_t)np * 4u * 2048u);
                for (int j = 0; j < np; ++j) {
                    const int pg = buf[min(8 * (int)tc + j, MAX_ITEM_PAGES - 1)];
                    const int yk = ((pg * 2 + 0) * a.nkv + tit.g) * 16;
                    const int yv = ((pg * 2 + 1) * a.nkv + tit.g) * 16;
                    tma_load_2d(kd + j * 2048, &tmKV, &kv_full[st], 0, yk);
                    tma_load_2d(kd + REGION + j * 2048, &tmKV, &kv_full[st], 64, yk);
                    tma_load_2d(vd + j * 2048, &tmKV, &kv_full[st], 0, yv);
                    tma_load_2d(vd + REGION + j * 2048, &tmKV, &kv_full[st], 64, yv);
                }
            }
            __syncwarp();
            ++cs;
            if (++tc == (uint32_t)tit.nch) {
                tc = 0;
                iter_next(tit, a, hi);
                ++tni;  // the prefetch cursor is on this item or the next: its page list is staged
            }
        }
        if (!ok && lane == 0) {
            // let the copies still in flight land before the CTA exits
            volatile int quiet = 0;
            for (uint32_t x = cs > (uint32_t)NS ? cs - NS : 0u; x < cs; ++x)
                mbar_wait(&kv_full[x % NS], (x / NS) & 1u, &quiet, nullptr);
            mbar_wait(&q_full[tni & 1u], (tni >> 1) & 1u, &quiet, nullptr);
        }
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
                    if (!valid) {
                        // V row of a key past the request: zero it so that 0 * garbage cannot occur
                        uint8_t* vrow = smem + (cs % NS) * KV_STAGE + 2 * REGION + (jl >> 4) * 2048 + (jl & 15) * 128;
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
