// Paged-KV attention of the serving iteration: GQA decode attention with split-KV,
// causal attention of the prefill chunk, and the split-KV merge.
//
// Decode attention is the memory-bound operation NanoFlow overlaps with the GEMMs of
// another nano-batch (README "Introduction"; arXiv abstract). Each decode request r
// reads ctx_len[r] + 1 keys and values of every KV head from its pages; one page of
// one KV head is a contiguous 16 x d bf16 block (pool layout
// [page][K|V][kv_head][16][d]), fetched by TMA (two 128-byte-swizzled 16 x 64 boxes
// for d = 128) into a 16-stage shared-memory ring by a producer warp. Four consumer
// warps each take every fourth page of a work item and run q . K^T and P . V on the
// tensor cores (mma.sync m16n8k16 with the G query heads of a KV head as the rows),
// with an online softmax in fp32 (exp2, scores pre-scaled by log2(e)/sqrt(d)). The
// four partial states are merged through shared memory in a fixed order.
//
// Work item = (request, KV split, KV head). A request's keys are cut into splits of
// kDecodeSplitPages pages; the split structure depends only on ctx_len, so results
// do not depend on how requests are grouped into nano-batches. Items of a launch are
// dealt to the persistent CTAs in contiguous, equal-count ranges.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace {

constexpr int DEC_WARPS = 8;  // independent streaming warps per CTA
__host__ __device__ constexpr int dec_wstages(int hd) { return hd == 128 ? 3 : 6; }  // 24 KB in flight per warp
constexpr int PRE_STAGES = 4;  // 128 KB for d = 128: one CTA per SM
constexpr int PRE_THREADS = 5 * 32;
constexpr int BOX_BYTES = 16 * 128;  // one 16-row x 64-col bf16 box

// Keep the low / high bf16 of a packed pair.
__device__ __forceinline__ uint32_t keep_pair(uint32_t v, bool lo, bool hi) {
    return (lo ? (v & 0xFFFFu) : 0u) | (hi ? (v & 0xFFFF0000u) : 0u);
}

__device__ __forceinline__ float quad_max(float x) {
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
    return x;
}
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

// Work-item table entry (built by decode_schedule_kernel):
//   x = request r, y = g | split << 8 | nsplit << 20, z = index in page_indices of the item's
//   first page, w = keys of the request (ctx_len + 1).
struct DecMeta {
    int r, g, split, nsplit, base, nkeys, np;
};

__device__ __forceinline__ DecMeta unpack_meta(int4 v, int split_pages) {
    DecMeta m;
    m.r = v.x;
    m.g = v.y & 0xFF;
    m.split = (v.y >> 8) & 0xFFF;
    m.nsplit = (v.y >> 20) & 0xFFF;
    m.base = v.z;
    m.nkeys = v.w;
    const int npages = (m.nkeys + 15) >> 4;
    m.np = v.x < 0 ? 0 : min(split_pages, npages - m.split * split_pages);
    return m;
}

// Q of the item's G heads as the B operand (k = d, n = 8 heads; heads >= G are zero):
// b0 = Q[head lane/4][d = 16 kk + 2 (lane%4) + {0,1}], b1 = the same at d + 8.
template <int KSTEPS>
__device__ __forceinline__ void load_q_frags(const DecodeArgs& a, const DecMeta& m, int lane, int hd,
                                             uint32_t (&qb)[KSTEPS][2]) {
    const int h = lane >> 2, c0 = (lane & 3) * 2;
    const bool ok = m.r >= 0 && h < a.G;
    const uint16_t* q0 = a.q + ((size_t)(m.r < 0 ? 0 : m.r) * a.nq + (size_t)m.g * a.G + (ok ? h : 0)) * hd;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
        qb[kk][0] = ok ? __ldg(reinterpret_cast<const unsigned int*>(q0 + kk * 16 + c0)) : 0u;
        qb[kk][1] = ok ? __ldg(reinterpret_cast<const unsigned int*>(q0 + kk * 16 + 8 + c0)) : 0u;
    }
}

__device__ __forceinline__ int load_page_ids(const DecodeArgs& a, const DecMeta& m, int lane) {
    int pg = 0;
    if (lane < m.np) {
        pg = __ldg(a.page_indices + m.base + lane);
        if (pg < 0 || pg >= a.num_pages) {
            set_status(a.status, NF_ERR_DEVICE_BOUNDS);
            pg = 0;
        }
    }
    return pg;
}

// max / sum over the 8 lanes that share lane % 4 (the 16 keys of a page, per head column)
__device__ __forceinline__ float col_max(float x) {
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
    return x;
}
__device__ __forceinline__ float col_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 16);
    return x;
}

// Each warp is an independent streaming pipeline: it owns NSTW ring stages (one page of
// one KV head, K and V, per stage), issues its own TMA loads (lane 0) and processes work
// items my_b + w, my_b + w + DEC_WARPS, ... Its page stream runs across item boundaries;
// the next item's table entry, page list and Q fragments are loaded while the current item
// streams, so no global-load latency sits between pages or between items.
//
// Per page (16 keys) the warp computes S^T = K Q^T (m16n8k16: keys as rows, the G query
// heads of the KV head as the 8 columns), an online softmax per head column, and
// O^T += V^T P^T (d as rows). P^T is turned from accumulator layout into operand layout
// with movmatrix. The running maximum is only moved when a page's maximum exceeds it by
// more than 2^8 (exponents stay <= 256), which skips most accumulator rescales.
template <int HD>
__global__ void __launch_bounds__(DEC_WARPS * 32, 1)
    decode_attention_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int BOXES = HD / 64;
    constexpr uint32_t KV_BYTES = BOXES * BOX_BYTES;  // one page, one KV head, K or V
    constexpr uint32_t STAGE_BYTES = 2 * KV_BYTES;
    constexpr int NSTW = dec_wstages(HD);
    constexpr int KSTEPS = HD / 16;
    constexpr int MT = HD / 16;  // m-tiles of O^T
    constexpr float LAZY = 8.0f;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_all = reinterpret_cast<uint64_t*>(smem + DEC_WARPS * NSTW * STAGE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t t_start = 0;
    if (threadIdx.x == 0) {
        t_start = globaltimer_ns();
        for (int s = 0; s < DEC_WARPS * NSTW; ++s) mbar_init(&full_all[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    const int ib = a.item_off[a.req_begin];
    const int ie = a.item_off[a.req_end];
    const int nitems = ie - ib;
    const int my_b = ib + (int)(((long long)nitems * blockIdx.x) / gridDim.x);
    const int my_e = ib + (int)(((long long)nitems * (blockIdx.x + 1)) / gridDim.x);

    uint8_t* wsm = smem + warp * NSTW * STAGE_BYTES;
    uint64_t* full = full_all + warp * NSTW;
    const uint32_t wsm_u32 = smem_u32(wsm);
    const int kr = lane >> 2;            // key row of the S^T fragment (and +8)
    const int hc = (lane & 3) * 2;       // head column pair of the S^T fragment
    const int4* tab = reinterpret_cast<const int4*>(a.item_tab);
    const int4 none = make_int4(-1, 0, 0, 0);

    int it = my_b + warp;
    DecMeta cur = unpack_meta(it < my_e ? __ldg(tab + it) : none, a.split_pages);
    DecMeta nxt = unpack_meta(it + DEC_WARPS < my_e ? __ldg(tab + it + DEC_WARPS) : none, a.split_pages);
    int4 tab_nn = it + 2 * DEC_WARPS < my_e ? __ldg(tab + it + 2 * DEC_WARPS) : none;
    uint32_t q_cur[KSTEPS][2], q_nxt[KSTEPS][2];
    load_q_frags<KSTEPS>(a, cur, lane, HD, q_cur);
    int pages_cur = load_page_ids(a, cur, lane);
    int pages_nxt = load_page_ids(a, nxt, lane);

    // issue cursor over the warp's page stream: src 0 = current item, 1 = next item, 2 = wait
    int iss_src = cur.np > 0 ? 0 : 2, iss_k = 0;
    uint32_t issued = 0, consumed = 0;
    volatile int quiet = 0;
    bool alive = true;

#define NF_DEC_TOP_UP()                                                                              \
    while (issued - consumed < (uint32_t)NSTW && iss_src < 2) {                                      \
        const DecMeta& im = iss_src == 0 ? cur : nxt;                                                \
        const int pg = __shfl_sync(0xffffffffu, iss_src == 0 ? pages_cur : pages_nxt, iss_k);        \
        if (lane == 0) {                                                                             \
            const int st = (int)(issued % NSTW);                                                     \
            uint8_t* dst = wsm + st * STAGE_BYTES;                                                   \
            fence_proxy_async_smem();                                                                \
            mbar_arrive_expect_tx(&full[st], STAGE_BYTES);                                           \
            const char* pgb = reinterpret_cast<const char*>(a.kv_pool) + (size_t)pg * 2 * a.nkv * 16 * HD * 2; \
            _Pragma("unroll") for (int b = 0; b < BOXES; ++b) {                                      \
                bulk_load(dst + b * BOX_BYTES, pgb + ((size_t)(0 * BOXES + b) * a.nkv + im.g) * BOX_BYTES, \
                          BOX_BYTES, &full[st]);                                                     \
                bulk_load(dst + KV_BYTES + b * BOX_BYTES,                                            \
                          pgb + ((size_t)(1 * BOXES + b) * a.nkv + im.g) * BOX_BYTES, BOX_BYTES, &full[st]); \
            }                                                                                        \
        }                                                                                            \
        ++issued;                                                                                    \
        if (++iss_k == im.np) {                                                                      \
            iss_k = 0;                                                                               \
            iss_src = (iss_src == 0 && nxt.np > 0) ? 1 : 2;                                          \
        }                                                                                            \
    }

    NF_DEC_TOP_UP();
    while (cur.np > 0 && alive) {
        load_q_frags<KSTEPS>(a, nxt, lane, HD, q_nxt);  // prefetch for the next item

        float o[MT][4];
#pragma unroll
        for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;  // heads hc, hc + 1

        for (int p = 0; p < cur.np; ++p) {
            const int st = (int)(consumed % NSTW);
            const uint32_t phase = (consumed / NSTW) & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&full[st], phase, &quiet, a.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { alive = false; break; }
            const uint32_t sK = wsm_u32 + st * STAGE_BYTES;
            const uint32_t sV = sK + KV_BYTES;
            const int key0 = (cur.split * a.split_pages + p) * 16;
            const int nvalid = min(16, cur.nkeys - key0);

            // S^T[16 keys x 8 heads] = K Q^T, even and odd k-steps in two independent chains
            float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int mi = lane >> 3;
                const int key = (mi & 1) * 8 + (lane & 7);
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
                    const int dc = kk * 16 + (mi >> 1) * 8;
                    uint32_t ka[4];
                    ldmatrix_x4(sK + (dc / 64) * BOX_BYTES + sw128_offset(key, dc % 64), ka[0], ka[1], ka[2], ka[3]);
                    mma_16816((kk & 1) ? s2 : s, ka, q_cur[kk][0], q_cur[kk][1]);
                }
            }
            const bool v0 = kr < nvalid, v8 = kr + 8 < nvalid;
            s[0] = v0 ? (s[0] + s2[0]) * a.scale_log2 : -INFINITY;   // key kr, head hc
            s[1] = v0 ? (s[1] + s2[1]) * a.scale_log2 : -INFINITY;   // key kr, head hc + 1
            s[2] = v8 ? (s[2] + s2[2]) * a.scale_log2 : -INFINITY;   // key kr + 8, head hc
            s[3] = v8 ? (s[3] + s2[3]) * a.scale_log2 : -INFINITY;   // key kr + 8, head hc + 1
            // the running maximum moves only if some score exceeds it by more than LAZY
            const float tA = fmaxf(s[0], s[2]), tB = fmaxf(s[1], s[3]);
            if (__any_sync(0xffffffffu, tA > mA + LAZY || tB > mB + LAZY)) {
                const float xA = col_max(tA), xB = col_max(tB);
                const float nA = softmax_max_update(mA, xA), nB = softmax_max_update(mB, xB);
                const float cA = softmax_rescale(mA, nA), cB = softmax_rescale(mB, nB);
                mA = nA;
                mB = nB;
                lA *= cA;
                lB *= cB;
#pragma unroll
                for (int i = 0; i < MT; ++i) { o[i][0] *= cA; o[i][1] *= cB; o[i][2] *= cA; o[i][3] *= cB; }
            }
            s[0] = exp2f(s[0] - mA);
            s[1] = exp2f(s[1] - mB);
            s[2] = exp2f(s[2] - mA);
            s[3] = exp2f(s[3] - mB);
            lA += s[0] + s[2];
            lB += s[1] + s[3];
            // P^T as the B operand (k = keys, n = heads)
            const uint32_t pb0 = movmatrix_trans(pack_bf16x2(s[0], s[1]));
            const uint32_t pb1 = movmatrix_trans(pack_bf16x2(s[2], s[3]));

            // O^T[d x 8 heads] += V^T P^T; V rows of keys past the request are zeroed
            const int kb = (lane & 3) * 2;
            const bool k0 = kb < nvalid, k1 = kb + 1 < nvalid, k8 = kb + 8 < nvalid, k9 = kb + 9 < nvalid;
            {
                const int mi = lane >> 3;
                const int key = (mi >> 1) * 8 + (lane & 7);
#pragma unroll
                for (int i = 0; i < MT; ++i) {
                    const int dc = i * 16 + (mi & 1) * 8;
                    uint32_t va[4];
                    ldmatrix_x4_trans(sV + (dc / 64) * BOX_BYTES + sw128_offset(key, dc % 64), va[0], va[1], va[2],
                                      va[3]);
                    if (nvalid < 16) {
                        va[0] = keep_pair(va[0], k0, k1); va[1] = keep_pair(va[1], k0, k1);
                        va[2] = keep_pair(va[2], k8, k9); va[3] = keep_pair(va[3], k8, k9);
                    }
                    mma_16816(o[i], va, pb0, pb1);
                }
            }
            __syncwarp();
            ++consumed;
            NF_DEC_TOP_UP();  // refills the stage just released (at most one page)
        }
        if (!alive) break;
        // ---- item output: final (single split) or a split partial for the merge kernel
        lA = col_sum(lA);
        lB = col_sum(lB);
        const float iA = 1.f / lA, iB = 1.f / lB;
        const bool okA = hc < a.G, okB = hc + 1 < a.G;
        const size_t hA = (size_t)cur.g * a.G + hc;
        if (cur.nsplit == 1) {
            uint16_t* ob = a.out + (size_t)cur.r * a.nq * HD;
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                const int d0 = i * 16 + kr;
                if (okA) { ob[hA * HD + d0] = f2bf(o[i][0] * iA); ob[hA * HD + d0 + 8] = f2bf(o[i][2] * iA); }
                if (okB) { ob[(hA + 1) * HD + d0] = f2bf(o[i][1] * iB); ob[(hA + 1) * HD + d0 + 8] = f2bf(o[i][3] * iB); }
            }
        } else {
            float* po = a.part_o + (size_t)it * a.G * HD;
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                const int d0 = i * 16 + kr;
                if (okA) { po[(size_t)hc * HD + d0] = o[i][0] * iA; po[(size_t)hc * HD + d0 + 8] = o[i][2] * iA; }
                if (okB) { po[(size_t)(hc + 1) * HD + d0] = o[i][1] * iB; po[(size_t)(hc + 1) * HD + d0 + 8] = o[i][3] * iB; }
            }
            if (kr == 0) {
                if (okA) a.part_lse[(size_t)it * a.G + hc] = mA + log2f(lA);
                if (okB) a.part_lse[(size_t)it * a.G + hc + 1] = mB + log2f(lB);
            }
            // The warp that writes the last split of (r, g) merges all splits in split order.
            // Each launch adds exactly nsplit arrivals per (r, g), so counters need no reset
            // between the layers of an iteration.
            __threadfence();
            __syncwarp();
            int last = 0;
            if (lane == 0)
                last = (atomicAdd(a.merge_cnt + (size_t)cur.r * a.nkv + cur.g, 1) + 1) % cur.nsplit == 0;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                __threadfence();
                const int base = it - cur.split * a.nkv;  // item of split 0
                for (int e = lane; e < a.G * HD; e += 32) {
                    const int row = e / HD, col = e - row * HD;
                    float M = -INFINITY;
                    for (int sp = 0; sp < cur.nsplit; ++sp)
                        M = fmaxf(M, __ldcg(a.part_lse + (size_t)(base + sp * a.nkv) * a.G + row));
                    float L = 0.f, acc = 0.f;
                    for (int sp = 0; sp < cur.nsplit; ++sp) {
                        const size_t itm = (size_t)(base + sp * a.nkv);
                        const float w = exp2f(__ldcg(a.part_lse + itm * a.G + row) - M);
                        L += w;
                        acc += w * __ldcg(a.part_o + (itm * a.G + row) * HD + col);
                    }
                    a.out[((size_t)cur.r * a.nq + (size_t)cur.g * a.G + row) * HD + col] = f2bf(acc / L);
                }
            }
        }
        // ---- rotate: next item becomes current
        it += DEC_WARPS;
        cur = nxt;
        pages_cur = pages_nxt;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) { q_cur[kk][0] = q_nxt[kk][0]; q_cur[kk][1] = q_nxt[kk][1]; }
        nxt = unpack_meta(tab_nn, a.split_pages);
        pages_nxt = load_page_ids(a, nxt, lane);
        tab_nn = it + 2 * DEC_WARPS < my_e ? __ldg(tab + it + 2 * DEC_WARPS) : none;
        // the cursor was on the old next item (now current) or had issued all of it
        if (iss_src == 1) {
            iss_src = 0;
        } else {
            iss_src = nxt.np > 0 ? 1 : 2;
            iss_k = 0;
        }
        NF_DEC_TOP_UP();
    }
#undef NF_DEC_TOP_UP
    if (!alive && lane == 0) {
        // let this warp's copies still in flight land before the CTA exits
        for (uint32_t sq = consumed; sq < issued; ++sq)
            mbar_wait(&full[sq % NSTW], (sq / NSTW) & 1u, &quiet, nullptr);
    }
    __syncwarp();
    __syncthreads();
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

// ------------------------------------------------------------------ prefill chunk
// Work item = (q tile of 64 chunk rows, query head); K/V tiles of 64 keys (4 pages)
// stream through a 3-stage ring filled by a producer warp; four consumer warps own
// 16 query rows each. Causal: tile kt is needed by q tile qt iff kt <= qt.
template <int HD>
__global__ void __launch_bounds__(PRE_THREADS, 1)
    prefill_attention_kernel(const __grid_constant__ PrefillArgs a) {
    constexpr int BOXES = HD / 64;
    constexpr uint32_t PAGE_BYTES = BOXES * BOX_BYTES;      // one page of K (or V), one KV head
    constexpr uint32_t HALF_BYTES = 4 * PAGE_BYTES;          // 64 keys
    constexpr uint32_t STAGE_BYTES = 2 * HALF_BYTES;
    constexpr int KSTEPS = HD / 16;
    constexpr int NT = HD / 8;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + PRE_STAGES * STAGE_BYTES);
    uint64_t* empty = full + PRE_STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + PRE_STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t t_start = 0;
    if (threadIdx.x == 0) {
        t_start = globaltimer_ns();
        for (int s = 0; s < PRE_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 4); }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int C = a.prefill_len;
    const int nqt = (C + 63) / 64;
    const int nitems = nqt * a.nq;
    const int npages = (C + 15) >> 4;
    const int* pt = a.page_indices + a.page_indptr[a.num_decode];

    if (warp == 4) {
        if (lane == 0) {
            uint32_t seq = 0;
            bool ok = true;
            uint32_t outstanding = 0, parity_bits = 0;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
                const int qt = nqt - 1 - it / a.nq;
                const int h = it % a.nq;
                const int g = h / a.G;
                for (int kt = 0; kt <= qt; ++kt, ++seq) {
                    const int stage = (int)(seq % PRE_STAGES);
                    const uint32_t phase = (seq / PRE_STAGES) & 1u;
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
                    outstanding &= ~(1u << stage);
                    uint8_t* st = smem + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    for (int pp = 0; pp < 4; ++pp) {
                        // pages past the chunk repeat its last page: finite data under masked keys
                        int pidx = min(kt * 4 + pp, npages - 1);
                        int page = pt[pidx];
                        if (page < 0 || page >= a.num_pages) { set_status(a.status, NF_ERR_DEVICE_BOUNDS); page = 0; }
                        const char* pgb = reinterpret_cast<const char*>(a.kv_pool) + (size_t)page * 2 * a.nkv * 16 * HD * 2;
#pragma unroll
                        for (int b = 0; b < BOXES; ++b) {
                            bulk_load(st + pp * PAGE_BYTES + b * BOX_BYTES,
                                      pgb + ((size_t)(0 * BOXES + b) * a.nkv + g) * BOX_BYTES, BOX_BYTES, &full[stage]);
                            bulk_load(st + HALF_BYTES + pp * PAGE_BYTES + b * BOX_BYTES,
                                      pgb + ((size_t)(1 * BOXES + b) * a.nkv + g) * BOX_BYTES, BOX_BYTES, &full[stage]);
                        }
                    }
                    outstanding |= 1u << stage;
                    parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
                }
            }
            if (!ok) {
                volatile int quiet = 0;
                for (int st = 0; st < PRE_STAGES; ++st)
                    if (outstanding & (1u << st)) mbar_wait(&full[st], (parity_bits >> st) & 1u, &quiet, nullptr);
            }
        }
        __syncwarp();
    } else {
        const int qr = lane >> 2, qc = (lane & 3) * 2;
        uint32_t seq = 0;
        bool alive = true;
        for (int it = blockIdx.x; it < nitems && alive; it += gridDim.x) {
            const int qt = nqt - 1 - it / a.nq;
            const int h = it % a.nq;
            const int i0 = qt * 64 + warp * 16 + qr;  // chunk rows of this thread: i0, i0 + 8
            const int i1 = i0 + 8;
            uint32_t qa[KSTEPS][4];
            {
                const uint16_t* qb = a.q + (size_t)h * HD;
                const size_t rs = (size_t)a.nq * HD;
                const bool v0 = i0 < C, v1 = i1 < C;
                const uint16_t* q0 = qb + (size_t)(a.num_decode + i0) * rs;
                const uint16_t* q1 = qb + (size_t)(a.num_decode + i1) * rs;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
                    const int c = kk * 16 + qc;
                    qa[kk][0] = v0 ? *reinterpret_cast<const uint32_t*>(q0 + c) : 0u;
                    qa[kk][1] = v1 ? *reinterpret_cast<const uint32_t*>(q1 + c) : 0u;
                    qa[kk][2] = v0 ? *reinterpret_cast<const uint32_t*>(q0 + c + 8) : 0u;
                    qa[kk][3] = v1 ? *reinterpret_cast<const uint32_t*>(q1 + c + 8) : 0u;
                }
            }
            float o[NT][4];
#pragma unroll
            for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
            float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
            for (int kt = 0; kt <= qt; ++kt, ++seq) {
                const int stage = (int)(seq % PRE_STAGES);
                const uint32_t phase = (seq / PRE_STAGES) & 1u;
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&full[stage], phase, abort_flag, a.status) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) { alive = false; break; }
                const uint32_t sK = smem_u32(smem + stage * STAGE_BYTES);
                const uint32_t sV = sK + HALF_BYTES;
                float s[8][4];
#pragma unroll
                for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
                    for (int j = 0; j < 8; j += 2) {
                        const int mi = lane >> 3;
                        const int key = (j + (mi >> 1)) * 8 + (lane & 7);
                        const int dc = kk * 16 + (mi & 1) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4(sK + (key >> 4) * PAGE_BYTES + (dc / 64) * BOX_BYTES + sw128_offset(key & 15, dc % 64),
                                    b0, b1, b2, b3);
                        mma_16816(s[j], qa[kk], b0, b1);
                        mma_16816(s[j + 1], qa[kk], b2, b3);
                    }
                }
                const int kbase = kt * 64;
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int key = kbase + j * 8 + qc + e;
                        s[j][e] = (key <= i0) ? s[j][e] * a.scale_log2 : -INFINITY;
                        s[j][2 + e] = (key <= i1) ? s[j][2 + e] * a.scale_log2 : -INFINITY;
                        mx0 = fmaxf(mx0, s[j][e]);
                        mx1 = fmaxf(mx1, s[j][2 + e]);
                    }
                }
                mx0 = quad_max(mx0);
                mx1 = quad_max(mx1);
                const float mn0 = softmax_max_update(m0, mx0), mn1 = softmax_max_update(m1, mx1);
                // rows whose keys in this tile are all masked keep m = -inf: guard the rescale
                const float c0 = softmax_rescale(m0, mn0);
                const float c1 = softmax_rescale(m1, mn1);
                m0 = mn0;
                m1 = mn1;
                float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        s[j][e] = (mn0 == -INFINITY) ? 0.f : exp2f(s[j][e] - mn0);
                        s[j][2 + e] = (mn1 == -INFINITY) ? 0.f : exp2f(s[j][2 + e] - mn1);
                        ps0 += s[j][e];
                        ps1 += s[j][2 + e];
                    }
                }
                l0 = l0 * c0 + ps0;
                l1 = l1 * c1 + ps1;
#pragma unroll
                for (int j = 0; j < NT; ++j) { o[j][0] *= c0; o[j][1] *= c0; o[j][2] *= c1; o[j][3] *= c1; }
                // keys >= C (only in the last tile) get their V rows zeroed in the fragments
                const int kb = (lane & 3) * 2;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    uint32_t pa[4];
                    pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
                    pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
                    pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                    pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
                    const int key0 = kbase + kk * 16;
                    const bool tail = key0 + 16 > C;
                    const bool k0 = key0 + kb < C, k1 = key0 + kb + 1 < C;
                    const bool k8 = key0 + kb + 8 < C, k9 = key0 + kb + 9 < C;
#pragma unroll
                    for (int j = 0; j < NT; j += 2) {
                        const int mi = lane >> 3;
                        const int key = (mi & 1) * 8 + (lane & 7);
                        const int dc = j * 8 + (mi >> 1) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldmatrix_x4_trans(sV + kk * PAGE_BYTES + (dc / 64) * BOX_BYTES + sw128_offset(key, dc % 64),
                                          b0, b1, b2, b3);
                        if (tail) {
                            b0 = keep_pair(b0, k0, k1); b1 = keep_pair(b1, k8, k9);
                            b2 = keep_pair(b2, k0, k1); b3 = keep_pair(b3, k8, k9);
                        }
                        mma_16816(o[j], pa, b0, b1);
                        mma_16816(o[j + 1], pa, b2, b3);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
            }
            if (!alive) break;
            l0 = quad_sum(l0);
            l1 = quad_sum(l1);
            const float inv0 = 1.f / l0, inv1 = 1.f / l1;
            const size_t rs = (size_t)a.nq * HD;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const int c = j * 8 + qc;
                if (i0 < C) {
                    *reinterpret_cast<uint32_t*>(a.out + (size_t)(a.num_decode + i0) * rs + (size_t)h * HD + c) =
                        pack_bf16x2(o[j][0] * inv0, o[j][1] * inv0);
                }
                if (i1 < C) {
                    *reinterpret_cast<uint32_t*>(a.out + (size_t)(a.num_decode + i1) * rs + (size_t)h * HD + c) =
                        pack_bf16x2(o[j][2] * inv1, o[j][3] * inv1);
                }
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && a.trace != nullptr) {
        const int i = atomicAdd(a.trace_ctr, 1);
        if (i < a.trace_cap) {
            a.trace[i].kernel = NF_KERNEL_PREFILL_ATTN;
            a.trace[i].smid = (int32_t)smid();
            a.trace[i].t_start = t_start;
            a.trace[i].t_end = globaltimer_ns();
        }
    }
}

// Items per request: nkv * ceil(ceil((ctx+1)/16) / split_pages); exclusive prefix into item_off[0..R].
__global__ void decode_schedule_kernel(const int* ctx_len, int R, int nkv, int split_pages, int* item_off) {
    __shared__ int carry;
    __shared__ int warp_sums[32];
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < R; base += blockDim.x) {
        const int r = base + threadIdx.x;
        int v = 0;
        if (r < R) {
            const int npages = (ctx_len[r] + 1 + 15) >> 4;
            v = nkv * ((npages + split_pages - 1) / split_pages);
        }
        // block inclusive scan
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[w] = x;
        __syncthreads();
        if (w == 0) {
            const int nw = blockDim.x >> 5;
            int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            if (lane < nw) warp_sums[lane] = s;
        }
        __syncthreads();
        const int incl = x + (w > 0 ? warp_sums[w - 1] : 0);
        if (r < R) item_off[r] = carry + incl - v;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry += incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) item_off[R] = carry;
}

// Work-item table: items of request r are item_off[r] + split * nkv + g.
__global__ void decode_items_kernel(const int* ctx_len, const int* page_indptr, int R, int nkv, int split_pages,
                                    const int* item_off, int4* tab, int* merge_cnt) {
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
        const int nkeys = ctx_len[r] + 1;
        const int npages = (nkeys + 15) >> 4;
        const int nsplit = (npages + split_pages - 1) / split_pages;
        const int base = item_off[r];
        const int pbase = page_indptr[r];
        for (int sp = 0; sp < nsplit; ++sp)
            for (int g = 0; g < nkv; ++g)
                tab[base + sp * nkv + g] = make_int4(r, g | (sp << 8) | (nsplit << 20), pbase + sp * split_pages, nkeys);
        for (int g = 0; g < nkv; ++g) merge_cnt[(size_t)r * nkv + g] = 0;
    }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

int decode_smem_bytes(int hd) {
    const int stage = 2 * (hd / 64) * BOX_BYTES;
    return DEC_WARPS * dec_wstages(hd) * (stage + 8) + 1024;
}

int prefill_smem_bytes(int hd) {
    const int stage = 2 * 4 * (hd / 64) * BOX_BYTES;
    return PRE_STAGES * stage + 2 * PRE_STAGES * 8 + 16 + 1024;
}

cudaError_t launch_decode_schedule(const int* ctx_len, int R, int nkv, int split_pages, int* item_off,
                                   cudaStream_t stream) {
    decode_schedule_kernel<<<1, 1024, 0, stream>>>(ctx_len, R, nkv, split_pages, item_off);
    return cudaGetLastError();
}

cudaError_t launch_decode_items(const int* ctx_len, const int* page_indptr, int R, int nkv, int split_pages,
                                const int* item_off, void* item_tab, int* merge_cnt, cudaStream_t stream) {
    const int grid = (R + 255) / 256;
    if (grid <= 0) return cudaSuccess;
    decode_items_kernel<<<grid, 256, 0, stream>>>(ctx_len, page_indptr, R, nkv, split_pages, item_off,
                                                 reinterpret_cast<int4*>(item_tab), merge_cnt);
    return cudaGetLastError();
}

cudaError_t launch_decode_attention(const DecodeArgs& a, int head_dim, int grid, cudaStream_t stream) {
    if (grid <= 0 || a.req_end <= a.req_begin) return cudaSuccess;
    const int smem = decode_smem_bytes(head_dim);
    cudaError_t e;
    if (head_dim == 128) {
        static bool cfg = false;
        if (!cfg) { if ((e = set_smem(decode_attention_kernel<128>, smem)) != cudaSuccess) return e; cfg = true; }
        decode_attention_kernel<128><<<grid, DEC_WARPS * 32, smem, stream>>>(a);
    } else if (head_dim == 64) {
        static bool cfg = false;
        if (!cfg) { if ((e = set_smem(decode_attention_kernel<64>, smem)) != cudaSuccess) return e; cfg = true; }
        decode_attention_kernel<64><<<grid, DEC_WARPS * 32, smem, stream>>>(a);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_prefill_attention(const PrefillArgs& a, int head_dim, int grid, cudaStream_t stream) {
    if (grid <= 0 || a.prefill_len <= 0) return cudaSuccess;
    const int smem = prefill_smem_bytes(head_dim);
    cudaError_t e;
    if (head_dim == 128) {
        static bool cfg = false;
        if (!cfg) { if ((e = set_smem(prefill_attention_kernel<128>, smem)) != cudaSuccess) return e; cfg = true; }
        prefill_attention_kernel<128><<<grid, PRE_THREADS, smem, stream>>>(a);
    } else if (head_dim == 64) {
        static bool cfg = false;
        if (!cfg) { if ((e = set_smem(prefill_attention_kernel<64>, smem)) != cudaSuccess) return e; cfg = true; }
        prefill_attention_kernel<64><<<grid, PRE_THREADS, smem, stream>>>(a);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace nf

