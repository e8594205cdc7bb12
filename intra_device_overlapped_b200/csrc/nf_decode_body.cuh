// Paged GQA decode attention on the 5th-generation tensor cores as device functions: shared by the
// decode attention kernels (nf_decode_tc.cu, which describes the page layout, the split along KV and
// the roles) and by the persistent kernel that runs a whole layer (nf_mega.cu).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace decode_impl {

constexpr int ROWS = 128;                   // 8 KV heads x 16 keys of one page
constexpr uint32_t PAGE_BYTES = 65536;      // K and V of all heads of one page
constexpr uint32_t HALF_PAGE = 32768;       // K (or V) of all heads of one page
constexpr uint32_t REGION = 16384;          // one 64-column half of K or V: 128 rows x 128 B
constexpr float LAZY = 8.0f;
constexpr int kPrefetchPages = 4;           // L2 prefetch distance of the page loader
constexpr int ITEM_SLOTS = 4;               // work-item ring between the page loader and the other roles
constexpr int ITEM_READERS = 7;             // Q loader, two MMA issuers, four softmax warps

template <int NQ>
struct TcCfg {
    static constexpr int NSP = 3;                         // page stages (K and V, released after P V)
    static constexpr int NSB = 3;                         // S^T buffers in TMEM
    // P buffers: the softmax of page c writes buffer c % NPB once the P V of page c - NPB is done (one
    // buffer with 64 query heads, where three would not fit beside three page stages)
    static constexpr int NPB = NQ <= 32 ? 3 : 1;
    static constexpr uint32_t QB = NQ * 256;              // Q: two halves of NQ rows x 128 B
    static constexpr uint32_t PB = NQ * 256;              // P buffer: two key halves of NQ rows x 128 B
    static constexpr uint32_t OFF_Q = NSP * PAGE_BYTES;
    static constexpr uint32_t OFF_P = OFF_Q + QB;
    static constexpr uint32_t OFF_CF = OFF_P + NPB * PB;  // float[NQ] rescale factors / row sums
    static constexpr uint32_t OFF_BAR = OFF_CF + NQ * 4;
    static constexpr uint32_t OFF_RING = OFF_BAR + 40 * 8;   // int2[ITEM_SLOTS]: the CTA's work items
    static constexpr uint32_t SMEM = OFF_RING + ITEM_SLOTS * 8 + 1024;
    static constexpr uint32_t O_COL = NSB * NQ;           // O^T accumulator after the S^T buffers
    static constexpr uint32_t TMEM_COLS = (NSB + 1) * NQ <= 128 ? 128 : 256;
    static constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(128, NQ);
    static constexpr uint32_t IDESC_PV = umma_idesc_bf16_f32_amn(128, NQ);
    static_assert(SMEM <= 232448, "shared memory");
    static_assert((NSB + 1) * NQ <= 256, "tensor memory");
    // page_full / stage_free per stage, q_full, q_empty, s_full / s_free per S buffer, p_full / pv_done
    // per P buffer, o_free, drain, item_full / item_empty per ring slot
    static constexpr int BARRIERS = 2 * NSP + 2 + 2 * NSB + 2 * NPB + 2 + 2 * ITEM_SLOTS;
    static_assert(BARRIERS + 1 <= 40, "barrier slots (+1 for the TMEM slot and abort flag)");
};

// warp 0 loads whole pages (one bulk copy each), warp 1 issues the S^T MMAs and owns TMEM, warps 2..5
// run the softmax, warp 6 loads each item's Q (TMA) once the previous item's scores are done, so that
// the page ring keeps streaming across item boundaries, and warp 7 issues the P V MMAs
constexpr int THREADS = 256;

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Walks the CTA's work items: chunks whose first page (in the page prefix of the requests) lies
// in [lo, hi). A request of npages pages has nch = ceil(npages / chunk_pages) chunks; chunk c holds
// pages [c npages / nch, (c + 1) npages / nch).
struct ItemIter {
    int r, c;            // request, chunk
    int nkeys, npages;   // of the request
    int nch;
    int pg0, pg1;        // the chunk's pages [pg0, pg1) within the request
    long long start;     // prefix position of the chunk's first page
    bool valid;
};

__device__ __forceinline__ void item_req(ItemIter& it, const DecodeArgs& a) {
    it.nkeys = max(a.ctx_len[it.r], 0) + 1;
    it.npages = (it.nkeys + 15) >> 4;
    it.nch = ceil_div(it.npages, a.split_pages);
}

__device__ __forceinline__ void item_chunk(ItemIter& it, const DecodeArgs& a, long long hi) {
    it.pg0 = (int)((long long)it.c * it.npages / it.nch);
    it.pg1 = (int)((long long)(it.c + 1) * it.npages / it.nch);
    it.start = (long long)a.item_off[it.r] + it.pg0;
    it.valid = it.r < a.req_end && it.start < hi;
}

__device__ __forceinline__ void item_init(ItemIter& it, const DecodeArgs& a, long long lo, long long hi) {
    int low = a.req_begin, high = a.req_end - 1;
    while (low < high) {  // last request whose first page is at or before lo
        const int mid = (low + high + 1) >> 1;
        if ((long long)a.item_off[mid] <= lo) low = mid; else high = mid - 1;
    }
    it.r = low;
    item_req(it, a);
    const long long off = lo - (long long)a.item_off[it.r];
    // first chunk starting at or after lo: c n / nch >= off  <=>  c >= off nch / n
    it.c = off > 0 ? (int)((off * it.nch + it.npages - 1) / it.npages) : 0;
    if (it.c >= it.nch) {
        it.r += 1;
        it.c = 0;
        if (it.r < a.req_end) item_req(it, a);
    }
    if (it.r < a.req_end) item_chunk(it, a, hi); else it.valid = false;
}

__device__ __forceinline__ void item_next(ItemIter& it, const DecodeArgs& a, long long hi) {
    if (++it.c == it.nch) {
        it.c = 0;
        if (++it.r >= a.req_end) { it.valid = false; return; }
        item_req(it, a);
    }
    item_chunk(it, a, hi);
}

// The item (request r, chunk c), all fields set.
__device__ __forceinline__ void item_set(ItemIter& it, const DecodeArgs& a, int r, int c) {
    it.r = r;
    it.c = c;
    item_req(it, a);
    it.pg0 = (int)((long long)c * it.npages / it.nch);
    it.pg1 = (int)((long long)(c + 1) * it.npages / it.nch);
    it.start = (long long)a.item_off[r] + it.pg0;
    it.valid = true;
}

// Global item k of the launch (items of requests [req_begin, req_end) in request order, chunks in
// order) as (request, chunk).
__device__ __forceinline__ int2 item_of(const DecodeArgs& a, long long k) {
    if (a.chunk_off == nullptr) return make_int2((int)k, 0);   // one chunk per request
    int low = a.req_begin, high = a.req_end - 1;
    while (low < high) {  // last request whose first chunk is at or before k
        const int mid = (low + high + 1) >> 1;
        if ((long long)a.chunk_off[mid] <= k) low = mid; else high = mid - 1;
    }
    return make_int2(low, (int)(k - a.chunk_off[low]));
}

// The work items of a CTA pass from the page loader to the other roles through a ring of ITEM_SLOTS
// (request, chunk) pairs ((-1, 0) ends the sequence): item_full[s] completes when the loader has
// written slot s, item_empty[s] when all ITEM_READERS warps have read it.
struct ItemRing {
    int2* slot;
    uint64_t* full;
    uint64_t* empty;
};

// Reader side: the ni-th item of the CTA into `it` (valid = false at the end of the sequence).
// Returns false if the wait gave up (the abort flag is then raised).
__device__ __forceinline__ bool ring_get(const ItemRing& ring, const DecodeArgs& a, uint32_t ni, ItemIter& it,
                                         volatile int* abort_flag, int lane) {
    const uint32_t s = ni % ITEM_SLOTS;
    const uint32_t par = (ni / ITEM_SLOTS) & 1u;
    int ok = 1;
    if (!__all_sync(0xffffffffu, mbar_test_wait(smem_u32(&ring.full[s]), par)))
        if (lane == 0) ok = mbar_wait(&ring.full[s], par, abort_flag, a.status) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) { it.valid = false; return false; }
    const volatile int* vs = reinterpret_cast<volatile int*>(&ring.slot[s]);
    const int2 v = make_int2(vs[0], vs[1]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring.empty[s]);
    if (v.x < 0) it.valid = false; else item_set(it, a, v.x, v.y);
    return true;
}

// Position in the CTA's page sequence: page j (within the request) of the current item, cs-th page
// overall, ni-th item.
struct PageCursor {
    ItemIter it;
    int j;
    uint32_t cs, ni;
    bool valid;
};

__device__ __forceinline__ void cursor_init(PageCursor& x, const DecodeArgs& a, const ItemRing& ring,
                                            volatile int* abort_flag, int lane) {
    x.cs = 0;
    x.ni = 0;
    ring_get(ring, a, 0, x.it, abort_flag, lane);
    x.j = x.it.pg0;
    x.valid = x.it.valid;
}

__device__ __forceinline__ void cursor_next(PageCursor& x, const DecodeArgs& a, const ItemRing& ring,
                                            volatile int* abort_flag, int lane) {
    ++x.cs;
    if (++x.j == x.it.pg1) {
        ++x.ni;
        ring_get(ring, a, x.ni, x.it, abort_flag, lane);
        x.j = x.it.pg0;
        x.valid = x.it.valid;
    }
}

// Non-blocking: has the phase of `bar` with this parity completed? (uniform across the warp)
// (test_wait returns at once; try_wait may hold the thread for a while before it reports an
// incomplete phase, which would keep the issuer from work that is ready elsewhere)
__device__ __forceinline__ bool test_bcast(uint64_t* bar, uint32_t parity, int lane) {
    int ok = 0;
    if (lane == 0) ok = mbar_test_wait(smem_u32(bar), parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ bool wait_bcast(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                           int lane) {
    // fast path: every lane tests the (usually already completed) phase; a completed phase stays
    // completed until this warp moves on, so the lanes agree once all have seen it
    if (__all_sync(0xffffffffu, mbar_test_wait(smem_u32(bar), parity))) return true;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// One CTA's part of a decode attention launch (256 threads, all in a role). `smem`: the
// 1024-byte-aligned dynamic shared memory (TcCfg<NQ>::SMEM - 1024 bytes are used); `tmem`: a TMEM
// allocation of at least TcCfg<NQ>::TMEM_COLS columns that the caller owns. Without a claim counter
// CTA `cta` of `ncta` walks its equal share of the launch's page prefix. The body starts and ends on
// a block-wide barrier and invalidates every mbarrier it initialised before it returns.
template <int NQ>
__device__ __forceinline__ void decode_body(const CUtensorMap* tmQ, const DecodeArgs& a, uint8_t* smem, uint32_t tmem,
                                            int cta, int ncta) {
    using C = TcCfg<NQ>;
    constexpr int NSP = C::NSP, NSB = C::NSB, NPB = C::NPB;
    constexpr int G = NQ / 8;
    float* cfs = reinterpret_cast<float*>(smem + C::OFF_CF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* page_full = bars;                // [NSP] the page's bulk copy has landed
    uint64_t* stage_free = page_full + NSP;    // [NSP] the P V of the stage's page has completed
    uint64_t* q_full = stage_free + NSP;       // [1]
    uint64_t* q_empty = q_full + 1;            // [1]
    uint64_t* s_full = q_empty + 1;            // [NSB]
    uint64_t* s_free = s_full + NSB;           // [NSB]
    uint64_t* p_full = s_free + NSB;           // [NPB]
    uint64_t* pv_done = p_full + NPB;          // [NPB]
    uint64_t* o_free = pv_done + NPB;          // [1]
    uint64_t* drain = o_free + 1;              // [1]
    uint64_t* item_full = drain + 1;           // [ITEM_SLOTS]
    uint64_t* item_empty = item_full + ITEM_SLOTS;  // [ITEM_SLOTS]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_empty + ITEM_SLOTS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const ItemRing ring{reinterpret_cast<int2*>(smem + C::OFF_RING), item_full, item_empty};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // P buffers start at zero: only the block-diagonal entries are ever written
    for (uint32_t i = threadIdx.x; i < NPB * C::PB / 16; i += THREADS)
        reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NSP; ++i) { mbar_init(&page_full[i], 1); mbar_init(&stage_free[i], 1); }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < NPB; ++i) { mbar_init(&p_full[i], 4); mbar_init(&pv_done[i], 1); }
        for (int i = 0; i < NSB; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 4); }
        mbar_init(o_free, 4);
        mbar_init(drain, 2);
        for (int i = 0; i < ITEM_SLOTS; ++i) { mbar_init(&item_full[i], 1); mbar_init(&item_empty[i], ITEM_READERS); }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(tmQ);
    }
    fence_proxy_async_smem();  // zeroed P buffers -> tensor-core reads
    __syncthreads();
    const uint32_t sbase = smem_u32(smem);

    const long long W0 = a.item_off[a.req_begin];
    const long long W = (long long)a.item_off[a.req_end] - W0;
    const long long lo = W0 + W * cta / ncta;
    const long long hi = W0 + W * (cta + 1) / ncta;

    if (warp == 6) {
        // ---------------- Q loader: two 64-column halves of the item's NQ query rows (TMA)
        ItemIter it;
        uint32_t ni = 0;
        for (ring_get(ring, a, 0, it, abort_flag, lane); it.valid; ring_get(ring, a, ++ni, it, abort_flag, lane)) {
            if (!wait_bcast(q_empty, (ni & 1u) ^ 1u, abort_flag, a.status, lane)) break;
            if (lane == 0) {
                uint8_t* qd = smem + C::OFF_Q;
                mbar_arrive_expect_tx(q_full, C::QB);
                tma_load_2d(qd, tmQ, q_full, 0, it.r * NQ);
                tma_load_2d(qd + NQ * 128, tmQ, q_full, 64, it.r * NQ);
            }
            __syncwarp();
        }
        if (lane == 0 && ni > 0) {  // the last Q load lands before the CTA exits
            volatile int quiet = 0;
            mbar_wait(q_full, (ni - 1) & 1u, &quiet, nullptr);
        }
        __syncwarp();
    } else if (warp == 0) {
        // ---------------- page loader: one 64 KB bulk copy per page (K and V of all heads) into the
        // page ring. An SM completes bulk copies at a rate that hardly depends on their size, so whole
        // pages stream about twice as fast as separate K and V halves. Page ids are read 32 at a time
        // (one per lane) and handed to lane 0.
        //
        // The loader also chooses the CTA's work items and publishes them in the item ring just before
        // it loads their pages: with a claim counter it takes the launch's next item from it, so that
        // CTAs that run faster (SMs differ by more than 10% in the bandwidth they get) take more items
        // and all finish together; without one it walks its share [lo, hi) of the page prefix.
        uint64_t* full = page_full;
        uint8_t* pring = smem;
        ItemIter walk;
        if (a.claim_ctr == nullptr) item_init(walk, a, lo, hi);
        const long long k0 = a.chunk_off ? a.chunk_off[a.req_begin] : a.req_begin;
        const long long k1 = a.chunk_off ? a.chunk_off[a.req_end] : a.req_end;
        // the n-th item: chosen, published in the ring, and set in `it` (valid = false at the end)
        auto produce = [&](uint32_t n, ItemIter& it) -> bool {
            const uint32_t slot = n % ITEM_SLOTS;
            if (n >= (uint32_t)ITEM_SLOTS &&
                !wait_bcast(&item_empty[slot], ((n / ITEM_SLOTS) - 1u) & 1u, abort_flag, a.status, lane)) {
                it.valid = false;
                return false;
            }
            int2 v;
            if (a.claim_ctr != nullptr) {
                int kk = 0;
                if (lane == 0) kk = atomicAdd(a.claim_ctr, 1);
                const long long k = k0 + __shfl_sync(0xffffffffu, kk, 0);
                v = k < k1 ? item_of(a, k) : make_int2(-1, 0);
            } else {
                v = walk.valid ? make_int2(walk.r, walk.c) : make_int2(-1, 0);
                if (walk.valid) item_next(walk, a, hi);
            }
            if (lane == 0) {
                volatile int* vd = reinterpret_cast<volatile int*>(&ring.slot[slot]);
                vd[0] = v.x;
                vd[1] = v.y;
                mbar_arrive(&item_full[slot]);  // release: the slot's contents before the phase
            }
            __syncwarp();
            if (v.x < 0) it.valid = false; else item_set(it, a, v.x, v.y);
            return true;
        };
        ItemIter it;
        uint32_t cs = 0, ni = 0;
        bool ok = produce(0, it);
        const char* pool = reinterpret_cast<const char*>(a.kv_pool);
        // each page is read once per launch: stream it through L2 without displacing reused data
        const uint64_t stream_policy = l2_policy_evict_first();
        // page ids of the current window of 32 pages (one per lane) and of the next one
        auto load_id = [&](int jj, int base, int rowlen, int pg1) -> int {
            // an index past the request's row of the page table, or a page outside the pool, is
            // recorded and page 0 read in its place
            int id = 0;
            if (jj < pg1) {
                if (jj < rowlen) id = __ldg(a.page_indices + base + jj);
                if (jj >= rowlen || id < 0 || id >= a.num_pages) {
                    set_status(a.status, NF_ERR_DEVICE_BOUNDS);
                    id = 0;
                }
            }
            return id;
        };
        for (; it.valid && ok; ok = ok && produce(++ni, it)) {
            const int base = a.page_indptr[it.r];
            const int rowlen = a.page_indptr[it.r + 1] - base;
            int ids = 0, ids_next = 0, w0 = it.pg0;
            // id of page jj of the request, jj in [w0, w0 + 64) (warp-uniform jj)
            auto id_of = [&](int jj) -> int {
                const int x = __shfl_sync(0xffffffffu, ids, (jj - w0) & 31);
                const int y = __shfl_sync(0xffffffffu, ids_next, (jj - w0) & 31);
                return jj - w0 < 32 ? x : y;
            };
            for (int j = it.pg0; j < it.pg1; ++j, ++cs) {
                if (((j - it.pg0) & 31) == 0) {
                    w0 = j;
                    ids = load_id(j + lane, base, rowlen, it.pg1);
                    ids_next = load_id(j + 32 + lane, base, rowlen, it.pg1);
                    if (j == it.pg0) {
                        // the item's first pages, which no earlier copy prefetched
                        for (int k = 1; k < kPrefetchPages && j + k < it.pg1; ++k) {
                            const int pid = id_of(j + k);
                            if (lane == 0) prefetch_l2_bulk(pool + (size_t)pid * PAGE_BYTES, PAGE_BYTES);
                        }
                    }
                }
                const int pg = id_of(j);
                const int pf = j + kPrefetchPages < it.pg1 ? id_of(j + kPrefetchPages) : -1;
                const int st = (int)(cs % NSP);
                // the stage's previous page (cs - NSP) must be consumed: its P V has completed (and with
                // it the S^T issued before it)
                if (cs >= (uint32_t)NSP &&
                    !wait_bcast(&stage_free[st], ((cs / NSP) - 1u) & 1u, abort_flag, a.status, lane)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[st], PAGE_BYTES);
                    bulk_load_hint(pring + st * PAGE_BYTES, pool + (size_t)pg * PAGE_BYTES, PAGE_BYTES, &full[st],
                                   stream_policy);
                    // a stage is held from its copy to the P V of its page, about three times the copy's
                    // own latency: a page bound for the ring kPrefetchPages pages later is fetched into L2
                    // now, so that its copy finds it there
                    if (pf >= 0) prefetch_l2_bulk(pool + (size_t)pf * PAGE_BYTES, PAGE_BYTES);
                }
            }
        }
        if (lane == 0) {
            // let the copies still in flight land before the CTA exits
            volatile int quiet = 0;
            for (uint32_t x = cs > (uint32_t)NSP ? cs - NSP : 0u; x < cs; ++x)
                mbar_wait(&full[x % NSP], (x / NSP) & 1u, &quiet, nullptr);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 7) {
        // ---------------- MMA issuers: warp 1 the scores S^T, warp 7 the products P V. Each follows the
        // pages in order and one elected lane issues whatever is ready; descriptors are built once and
        // offset by constants. Issuing the two kinds from different threads keeps a P V from waiting
        // behind the issue of later pages' scores (its commit frees the page's stage for the next load);
        // a commit tracks only the MMAs of the thread that issues it, so each warp's commits are its own.
        // S^T of page c needs page c in the ring and a free S^T buffer, so it runs at most NSP pages
        // ahead of the P V that frees the stage and NSB pages ahead of the softmax.
        const bool is_s = warp == 1;
        PageCursor x;
        cursor_init(x, a, ring, abort_flag, lane);
        const uint64_t kd0 = umma_desc_sw128(sbase);
        const uint64_t qd0 = umma_desc_sw128(sbase + C::OFF_Q);
        const uint64_t vd0 = umma_desc_sw128_mn(sbase + HALF_PAGE, REGION, 1024);
        const uint64_t pd0 = umma_desc_sw128(sbase + C::OFF_P);
        auto issue_s = [&](const PageCursor& c) {
            const uint32_t st = c.cs % NSP, sb = c.cs % NSB;
            tc_fence_after();
            const uint64_t ad = kd0 + ((st * PAGE_BYTES) >> 4);
            const uint64_t bd = qd0;
            const uint32_t d = tmem + sb * NQ;
            if (elect_one()) {
                umma_bf16_c<false>(d, ad, bd, C::IDESC_S);
#pragma unroll
                for (int kk = 1; kk < 8; ++kk)
                    umma_bf16_c<true>(d, ad + (uint64_t)(((kk >> 2) * REGION + (kk & 3) * 32) >> 4),
                                      bd + (uint64_t)(((kk >> 2) * (NQ * 128) + (kk & 3) * 32) >> 4), C::IDESC_S);
                umma_commit(&s_full[sb]);
                if (c.j == c.it.pg1 - 1) umma_commit(q_empty);
            }
            __syncwarp();
        };
        auto issue_pv = [&](const PageCursor& c) {
            const uint32_t pb = c.cs % NPB, sv = c.cs % NSP;
            const bool first = c.j == c.it.pg0;
            tc_fence_after();
            const uint64_t ad = vd0 + ((sv * PAGE_BYTES) >> 4);
            const uint64_t bd = pd0 + ((pb * C::PB) >> 4);
            const uint32_t d = tmem + C::O_COL;
            if (elect_one()) {
                if (first) umma_bf16_c<false>(d, ad, bd, C::IDESC_PV);
                else umma_bf16_c<true>(d, ad, bd, C::IDESC_PV);
#pragma unroll
                for (int kk = 1; kk < ROWS / 16; ++kk)
                    umma_bf16_c<true>(d, ad + (uint64_t)((kk * 2048) >> 4),
                                      bd + (uint64_t)(((kk >> 2) * (NQ * 128) + (kk & 3) * 32) >> 4), C::IDESC_PV);
                umma_commit(&pv_done[pb]);
                umma_commit(&stage_free[sv]);
            }
            __syncwarp();
        };
        uint32_t idle = 0;      // polls since the last issue
        uint64_t idle_t0 = 0;   // time of the 64th of them
        while (x.valid) {
            const bool first = x.j == x.it.pg0;
            bool ready;
            if (is_s) {
                // its Q (first page of an item), its page and a free S^T buffer
                ready = (!first || test_bcast(q_full, x.ni & 1u, lane)) &&
                        test_bcast(&page_full[x.cs % NSP], (x.cs / NSP) & 1u, lane) &&
                        test_bcast(&s_free[x.cs % NSB], ((x.cs / NSB) & 1u) ^ 1u, lane);
            } else {
                // its probabilities (written after its S^T completed), and on an item's first page the
                // previous item's output read out of TMEM
                ready = test_bcast(&p_full[x.cs % NPB], (x.cs / NPB) & 1u, lane) &&
                        (!first || test_bcast(o_free, (x.ni & 1u) ^ 1u, lane));
            }
            if (ready) {
                if (is_s) issue_s(x); else issue_pv(x);
                cursor_next(x, a, ring, abort_flag, lane);
                idle = 0;
                continue;
            }
            // nothing ready: poll again, within the same time limit as every other wait (lane 0 decides
            // for the warp)
            if ((++idle & 63u) == 0) {
                int stop = 0;
                if (lane == 0) {
                    const uint64_t now = globaltimer_ns();
                    if (*abort_flag) {
                        stop = 1;
                    } else if (idle == 64) {
                        idle_t0 = now;
                    } else if (now - idle_t0 > NF_WAIT_LIMIT_NS) {
                        *abort_flag = 1;
                        set_status(a.status, NF_ERR_DEVICE_TIMEOUT);
                        stop = 1;
                    }
                }
                if (__shfl_sync(0xffffffffu, stop, 0)) break;
            }
        }
        // both issuers' MMAs have completed before TMEM is released (drain counts the two commits)
        if (elect_one()) umma_commit(drain);
        __syncwarp();
        if (lane == 0) {
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
        ItemIter it;
        uint32_t cs = 0, ni = 0;
        bool ok = true;
        // every softmax warp reads each item from the ring; the four agree on it before any named
        // barrier inside the item (a read that gave up in one warp ends the item loop in all four)
        auto next_item = [&](uint32_t n) {
            const bool got = ring_get(ring, a, n, it, abort_flag, lane);
            if (bar_red_or(4, 128, !got || !it.valid)) { it.valid = false; ok = ok && got; }
        };
        for (next_item(0); it.valid && ok; next_item(++ni)) {
            float m[G], lp[G];
#pragma unroll
            for (int i = 0; i < G; ++i) { m[i] = -INFINITY; lp[i] = 0.f; }
            for (int c = it.pg0; c < it.pg1; ++c, ++cs) {
                const uint32_t sb = cs % NSB;
                bool okc = wait_bcast(&s_full[sb], (cs / NSB) & 1u, abort_flag, a.status, lane);
                float sw[2 * G];  // scores of the warp's two heads' query columns
#pragma unroll
                for (int i = 0; i < 2 * G; ++i) sw[i] = -INFINITY;
                if (okc) {
                    tc_fence_after();
                    // the 2G score columns of this warp's two heads (constant indices in both
                    // branches keep tmp in registers)
                    float tmp[16];
                    tmem_ld16(tmem + lane_addr + sb * NQ + ((2 * q * G) & ~15), tmp);
                    if (((2 * q * G) & 15) != 0) {
#pragma unroll
                        for (int i = 0; i < 2 * G && i + 8 < 16; ++i) sw[i] = tmp[i + 8];
                    } else {
#pragma unroll
                        for (int i = 0; i < 2 * G; ++i) sw[i] = tmp[i];
                    }
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
                        const float nm = softmax_max_update(m[i], x);
                        cf[i] = softmax_rescale(m[i], nm);
                        m[i] = nm;
                        lp[i] *= cf[i];
                    }
                    if (c > it.pg0) {
                        if (k == 0) {
#pragma unroll
                            for (int i = 0; i < G; ++i) cfs[h * G + i] = cf[i];
                        }
                        bar_sync_n(2, 128);
                        // the previous page's P V must have landed in O^T before it is rescaled
                        okc = okc && wait_bcast(&pv_done[(cs - 1) % NPB], ((cs - 1) / NPB) & 1u, abort_flag,
                                                a.status, lane);
                        if (okc) {
                            tc_fence_after();
#pragma unroll
                            for (int c16 = 0; c16 < NQ / 16; ++c16) {
                                float o[16];
                                tmem_ld16(tmem + lane_addr + C::O_COL + c16 * 16, o);
#pragma unroll
                                for (int i = 0; i < 16; ++i) o[i] *= cfs[c16 * 16 + i];
                                tmem_st16(tmem + lane_addr + C::O_COL + c16 * 16, o);
                            }
                            tc_fence_before();
                        }
                        bar_sync_n(2, 128);
                    }
                }
                // P entries of this row (its G query heads) into this page's P buffer
                const uint32_t pb = cs % NPB;
                if (cs >= (uint32_t)NPB)
                    okc = okc && wait_bcast(&pv_done[pb], ((cs - NPB) / NPB) & 1u, abort_flag, a.status, lane);
                if (okc) {
                    uint8_t* pbuf = smem + C::OFF_P + pb * C::PB + (t >> 6) * (NQ * 128);
#pragma unroll
                    for (int i = 0; i < G; ++i) {
                        const float p = exp2f(s[i] - m[i]);  // 0 for masked keys
                        lp[i] += p;
                        *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128_offset(h * G + i, t & 63)) =
                            __float2bfloat16_rn(p);
                    }
                    if ((it.nkeys & 15) != 0 && c == it.npages - 1) {  // CTA-uniform
                        // V rows of keys past the request in the last page: zero them so that
                        // 0 * garbage cannot occur in P V. One copy brings K and V of the page, and
                        // its S^T (which waited for that copy) has completed, so V has landed; the
                        // stage is refilled only after this page's P V.
                        if (okc && c * 16 + k >= it.nkeys) {
                            uint8_t* vrow = smem + (cs % NSP) * PAGE_BYTES + HALF_PAGE + t * 128;
#pragma unroll
                            for (int b = 0; b < 2; ++b)
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    reinterpret_cast<uint4*>(vrow + b * REGION)[i] = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && okc) mbar_arrive(&p_full[pb]);
                if (bar_red_or(3, 128, !okc)) { ok = false; break; }
            }
            if (!ok) break;
            // ---- item output: row sums per query head, then O^T (thread = one d); a request of one
            // chunk is normalised and written, a chunk of a longer request leaves its partial
            const bool single = it.nch == 1;
            const int slot = single ? 0 : a.chunk_off[it.r] + it.c;
#pragma unroll
            for (int i = 0; i < G; ++i) {
                float x = lp[i];
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (k == 0) {
                    if (single) {
                        cfs[h * G + i] = x;
                    } else {
                        a.part_ml[((size_t)slot * NQ + h * G + i) * 2] = m[i];
                        a.part_ml[((size_t)slot * NQ + h * G + i) * 2 + 1] = x;
                    }
                }
            }
            bool okc = wait_bcast(&pv_done[(cs - 1) % NPB], ((cs - 1) / NPB) & 1u, abort_flag, a.status, lane);
            bar_sync_n(2, 128);
            if (okc) tc_fence_after();
#pragma unroll
            for (int c16 = 0; c16 < NQ / 16; ++c16) {
                float o[16];
                if (okc) {
                    tmem_ld16(tmem + lane_addr + C::O_COL + c16 * 16, o);
                    if (single) {
                        uint16_t* ob = a.out + (size_t)it.r * NQ * 128 + t;  // thread t writes d = t of every head
#pragma unroll
                        for (int i = 0; i < 16; ++i) ob[(size_t)(c16 * 16 + i) * 128] = f2bf(o[i] / cfs[c16 * 16 + i]);
                    } else {
                        float* po = a.part_o + (size_t)slot * NQ * 128 + t;
#pragma unroll
                        for (int i = 0; i < 16; ++i) po[(size_t)(c16 * 16 + i) * 128] = o[i];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && okc) mbar_arrive(o_free);
            if (bar_red_or(2, 128, !okc)) { ok = false; break; }
        }
    }

    __syncthreads();
    if (threadIdx.x == 0)
        for (int i = 0; i < C::BARRIERS; ++i) mbar_inval(bars + i);
}

// Requests cut into several chunks: out = bf16(sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c) per
// query head, M the largest chunk maximum, both sums in chunk order (every factor is an exact power of
// two). One warp merges query heads [h0, h0 + MERGE_HEADS) of request r: lane l owns d = 4 l .. 4 l + 3
// (one 16-byte load per chunk and head), lane i < MERGE_HEADS finds M and the row sum of head h0 + i.
// A request of one chunk was written by the attention itself.
constexpr int MERGE_HEADS = 8;

template <int NQ>
__device__ __forceinline__ void merge_heads_warp(const DecodeArgs& a, int r, int h0, int lane) {
    const int npages = (max(a.ctx_len[r], 0) + 1 + 15) >> 4;
    const int nch = ceil_div(npages, a.split_pages);
    if (nch <= 1) return;
    const float* __restrict__ ml = a.part_ml + (size_t)a.chunk_off[r] * NQ * 2;
    const float* __restrict__ po = a.part_o + (size_t)a.chunk_off[r] * NQ * 128;
    float M = -INFINITY, L = 0.f;
    if (lane < MERGE_HEADS) {
        const int qh = h0 + lane;
        for (int c = 0; c < nch; ++c) M = fmaxf(M, ml[(c * NQ + qh) * 2]);
        for (int c = 0; c < nch; ++c) L += softmax_rescale(ml[(c * NQ + qh) * 2], M) * ml[(c * NQ + qh) * 2 + 1];
    }
    float Mh[MERGE_HEADS];
#pragma unroll
    for (int i = 0; i < MERGE_HEADS; ++i) Mh[i] = __shfl_sync(0xffffffffu, M, i);
    float acc[MERGE_HEADS][4];
#pragma unroll
    for (int i = 0; i < MERGE_HEADS; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    for (int c = 0; c < nch; ++c) {
        float4 v[MERGE_HEADS];
        float f[MERGE_HEADS];
#pragma unroll
        for (int i = 0; i < MERGE_HEADS; ++i) {
            v[i] = __ldcg(reinterpret_cast<const float4*>(po + ((size_t)c * NQ + h0 + i) * 128) + lane);
            f[i] = softmax_rescale(ml[(c * NQ + h0 + i) * 2], Mh[i]);
        }
#pragma unroll
        for (int i = 0; i < MERGE_HEADS; ++i) {
            acc[i][0] += f[i] * v[i].x;
            acc[i][1] += f[i] * v[i].y;
            acc[i][2] += f[i] * v[i].z;
            acc[i][3] += f[i] * v[i].w;
        }
    }
#pragma unroll
    for (int i = 0; i < MERGE_HEADS; ++i) {
        const float Li = __shfl_sync(0xffffffffu, L, i);
        *reinterpret_cast<uint2*>(a.out + ((size_t)r * NQ + h0 + i) * 128 + 4 * lane) =
            make_uint2((uint32_t)f2bf(acc[i][0] / Li) | ((uint32_t)f2bf(acc[i][1] / Li) << 16),
                       (uint32_t)f2bf(acc[i][2] / Li) | ((uint32_t)f2bf(acc[i][3] / Li) << 16));
    }
}

}  // namespace decode_impl
}  // namespace nf
