// Causal attention of the prefill chunk on the 5th-generation tensor cores (head dim 128) as a device
// function: shared by the prefill attention kernel (nf_prefill_tc.cu, which describes the method and
// the roles) and by the persistent kernel that runs a whole layer (nf_mega.cu).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nf_attention.h"
#include "nf_internal.h"
#include "nf_ptx.cuh"

namespace nf {
namespace prefill_impl {

constexpr int ROWS = 128;                     // query positions per unit
constexpr int KEYS = 128;                     // keys per key tile (8 pages of 16)
constexpr uint32_t HALF_TILE = 16384;         // 128 rows x 128 B: one 64-column half
constexpr uint32_t TILE = 2 * HALF_TILE;      // 128 rows x 128 columns of bf16
constexpr int NS = 2;                         // K stages and V stages (as many as S and P buffers)
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE;      // K stage s at OFF_K + s TILE
constexpr uint32_t OFF_V = OFF_K + NS * TILE; // V stage s at OFF_V + s TILE
constexpr uint32_t OFF_P = OFF_V + NS * TILE; // two P buffers
constexpr uint32_t OFF_BAR = OFF_P + 2 * TILE;
constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;           // S[2] at columns 0 / 128, O at 256
constexpr uint32_t O_COL = 256;
constexpr float LAZY = 8.0f;
constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(128, 128);
constexpr uint32_t IDESC_PV = umma_idesc_bf16_f32_bmn(128, 128);  // B (V) MN-major
static_assert(SMEM <= 232448, "shared memory");

// warp 0 loads Q (TMA) and K, warp 6 loads V (bulk copies), warp 1 issues MMAs and owns TMEM,
// warps 2..5 softmax and output (thread = query row). K stage x % NS is refilled once S of key
// tile x has completed, V stage x % NS once its P V has: the loaders wait on those barriers.
constexpr int THREADS = 224;

// Units are taken longest first (the last query tiles see the most keys) and dealt to the CTAs
// in a snake order, so the key tiles per CTA stay even.
__device__ __forceinline__ int unit_index(int k, int b, int grid) {
    return (k & 1) ? k * grid + (grid - 1 - b) : k * grid + b;
}

__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          int lane) {
    if (__all_sync(0xffffffffu, mbar_test_wait(smem_u32(bar), parity))) return true;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// mbarriers of the body: q_full, q_empty, k_full and v_full per stage, s_full, s_free, p_full and
// pv_done per buffer, o_free, drain
constexpr int BARRIERS = 2 + 2 * NS + 4 * 2 + 2;

// One CTA's part of a prefill attention launch: warps 0..6 take the roles above (further warps only
// join the two block-wide barriers). `smem`: the 1024-byte-aligned dynamic shared memory (SMEM - 1024
// bytes are used); `tmem`: a TMEM allocation of TMEM_COLS columns that the caller owns. CTA `cta` of
// `ncta` takes the units unit_index(k, cta, ncta), k = 0, 1, ... . The body starts and ends on a
// block-wide barrier and invalidates every mbarrier it initialised before it returns.
__device__ __forceinline__ void prefill_body(const CUtensorMap* tmQ, const PrefillArgs& a, uint8_t* smem, uint32_t tmem,
                                             int cta, int ncta) {
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* q_full = bars;              // [1]
    uint64_t* q_empty = q_full + 1;       // [1]
    uint64_t* k_full = q_empty + 1;       // [NS]
    uint64_t* v_full = k_full + NS;       // [NS]
    uint64_t* s_full = v_full + NS;       // [2]
    uint64_t* s_free = s_full + 2;        // [2]
    uint64_t* p_full = s_free + 2;        // [2]
    uint64_t* pv_done = p_full + 2;       // [2]
    uint64_t* o_free = pv_done + 2;       // [1]
    uint64_t* drain = o_free + 1;         // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < NS; ++i) { mbar_init(&k_full[i], 1); mbar_init(&v_full[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 4);
            mbar_init(&p_full[i], 4); mbar_init(&pv_done[i], 1);
        }
        mbar_init(o_free, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(tmQ);
    }
    __syncthreads();
    const uint32_t sbase = smem_u32(smem);

    const int C = a.prefill_len, R = a.num_decode, nq = a.nq, G = a.G;
    const int nqt = (C + ROWS - 1) / ROWS;            // query tiles
    const int units = nqt * nq;
    const int npages = (C + 15) >> 4;                 // pages of the chunk
    const int pbase = a.page_indptr[R];
    const size_t page_bytes = (size_t)a.nkv * 8192;   // K and V, two halves, nkv heads x 2 KB

    if (warp == 0 || warp == 6) {
        // ---------------- loaders: warp 0 Q and K, warp 6 V. Lanes 0..15 copy one 2 KB block
        // each: page i = lane % 8 of the tile, half b = lane / 8.
        const bool is_k = warp == 0;
        uint64_t* full = is_k ? k_full : v_full;
        uint8_t* ring = smem + (is_k ? OFF_K : OFF_V);
        const int b = (lane >> 3) & 1, i = lane & 7;
        const bool copier = lane < 16;
        uint32_t kt = 0, ni = 0;
        bool ok = true;
        for (int k = 0; ok; ++k, ++ni) {
            const int u = unit_index(k, cta, ncta);
            if (u >= units) break;
            const int h = u % nq, qt = nqt - 1 - u / nq, g = h / G;
            if (is_k) {
                if (!wait_warp(q_empty, (ni & 1u) ^ 1u, abort_flag, a.status, lane)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(q_full, TILE);
                    tma_load_3d(smem + OFF_Q, tmQ, q_full, 0, h, R + qt * ROWS);
                    tma_load_3d(smem + OFF_Q + HALF_TILE, tmQ, q_full, 64, h, R + qt * ROWS);
                }
            }
            for (int j = 0; j <= qt; ++j, ++kt) {
                const int st = (int)(kt % NS);
                // the page index is read before the stage wait so that its latency overlaps it
                const int pp = j * 8 + i;
                bool valid = copier && pp < npages;
                int pid = valid ? __ldg(a.page_indices + pbase + pp) : 0;
                if (kt >= (uint32_t)NS) {  // the stage's previous tile must be consumed: its S (K) or P V (V)
                    const uint32_t prev = kt - NS;
                    uint64_t* done = is_k ? &s_full[prev & 1u] : &pv_done[prev & 1u];
                    if (!wait_warp(done, (prev >> 1) & 1u, abort_flag, a.status, lane)) { ok = false; break; }
                }
                if (valid && (pid < 0 || pid >= a.num_pages)) { set_status(a.status, NF_ERR_DEVICE_BOUNDS); valid = false; }
                uint8_t* dst = ring + st * TILE + b * HALF_TILE + i * 2048;
                if (copier && !valid) {  // a page the chunk does not have: zero its rows
#pragma unroll 4
                    for (int c = 0; c < 128; ++c) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0u, 0u, 0u, 0u);
                    fence_proxy_async_smem();
                }
                const uint32_t nvalid = __popc(__ballot_sync(0xffffffffu, valid));
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(&full[st], nvalid * 2048u);
                __syncwarp();
                if (valid) {
                    const char* src = reinterpret_cast<const char*>(a.kv_pool) + (size_t)pid * page_bytes +
                                      (size_t)(((is_k ? 0 : 2) + b) * a.nkv + g) * 2048;
                    bulk_load(dst, src, 2048, &full[st]);
                }
            }
        }
        if (lane == 0) {
            volatile int quiet = 0;
            for (uint32_t x = kt > (uint32_t)NS ? kt - NS : 0u; x < kt; ++x)
                mbar_wait(&full[x % NS], (x / NS) & 1u, &quiet, nullptr);
            if (is_k && ni > 0) mbar_wait(q_full, (ni - 1) & 1u, &quiet, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (whole warp follows, one elected lane issues)
        const uint64_t qd = umma_desc_sw128(sbase + OFF_Q);
        const uint64_t kd0 = umma_desc_sw128(sbase + OFF_K);
        const uint64_t vd0 = umma_desc_sw128_mn(sbase + OFF_V, HALF_TILE, 1024);
        const uint64_t pd0 = umma_desc_sw128(sbase + OFF_P);
        uint32_t kt = 0, ni = 0;
        bool ok = true;
        auto issue_pv = [&](uint32_t x, bool first, uint32_t unit_no) -> bool {
            const uint32_t pb = x & 1u, st = x % NS;
            if (!wait_warp(&p_full[pb], (x >> 1) & 1u, abort_flag, a.status, lane)) return false;
            if (!wait_warp(&v_full[st], (x / NS) & 1u, abort_flag, a.status, lane)) return false;
            if (first && !wait_warp(o_free, (unit_no & 1u) ^ 1u, abort_flag, a.status, lane)) return false;
            tc_fence_after();
            const uint64_t ad = pd0 + ((pb * TILE) >> 4);
            const uint64_t bd = vd0 + ((st * TILE) >> 4);
            const uint32_t d = tmem + O_COL;
            if (elect_one()) {
                if (first) umma_bf16_c<false>(d, ad, bd, IDESC_PV);
                else umma_bf16_c<true>(d, ad, bd, IDESC_PV);
#pragma unroll
                for (int kk = 1; kk < KEYS / 16; ++kk)
                    umma_bf16_c<true>(d, ad + (uint64_t)(((kk >> 2) * HALF_TILE + (kk & 3) * 32) >> 4),
                                      bd + (uint64_t)((kk * 2048) >> 4), IDESC_PV);
                umma_commit(&pv_done[pb]);
            }
            __syncwarp();
            return true;
        };
        for (int k = 0; ok; ++k, ++ni) {
            const int u = unit_index(k, cta, ncta);
            if (u >= units) break;
            const int qt = nqt - 1 - u / nq;
            if (!wait_warp(q_full, ni & 1u, abort_flag, a.status, lane)) { ok = false; break; }
            for (int j = 0; j <= qt; ++j) {
                const uint32_t x = kt + j, st = x % NS, sb = x & 1u;
                if (!wait_warp(&k_full[st], (x / NS) & 1u, abort_flag, a.status, lane) ||
                    !wait_warp(&s_free[sb], ((x >> 1) & 1u) ^ 1u, abort_flag, a.status, lane)) { ok = false; break; }
                tc_fence_after();
                const uint64_t bd = kd0 + ((st * TILE) >> 4);
                const uint32_t d = tmem + sb * 128;
                if (elect_one()) {
                    umma_bf16_c<false>(d, qd, bd, IDESC_S);
#pragma unroll
                    for (int kk = 1; kk < 8; ++kk) {
                        const uint64_t off = (uint64_t)(((kk >> 2) * HALF_TILE + (kk & 3) * 32) >> 4);
                        umma_bf16_c<true>(d, qd + off, bd + off, IDESC_S);
                    }
                    umma_commit(&s_full[sb]);
                    if (j == qt) umma_commit(q_empty);
                }
                __syncwarp();
                if (j > 0 && !issue_pv(x - 1, j == 1, ni)) { ok = false; break; }
            }
            if (!ok) break;
            if (!issue_pv(kt + qt, qt == 0, ni)) { ok = false; break; }
            kt += qt + 1;
        }
        if (elect_one()) umma_commit(drain);
        __syncwarp();
        if (lane == 0) {
            volatile int quiet = 0;
            mbar_wait(drain, 0, &quiet, nullptr);
        }
        __syncwarp();
    } else if (warp < THREADS / 32) {
        // ---------------- softmax + output: thread = query row r of the unit
        const int qw = warp & 3;
        const int r = qw * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(qw * 32) << 16;
        uint32_t kt = 0, ni = 0;
        bool ok = true;
        for (int k = 0; ok; ++k, ++ni) {
            const int u = unit_index(k, cta, ncta);
            if (u >= units) break;
            const int h = u % nq, qt = nqt - 1 - u / nq;
            const int pos = qt * ROWS + r;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j <= qt && ok; ++j) {
                const uint32_t x = kt + j, sb = x & 1u, pb = x & 1u, st = x % NS;
                const bool diag = j == qt;
                if (!wait_warp(&s_full[sb], (x >> 1) & 1u, abort_flag, a.status, lane)) { ok = false; break; }
                tc_fence_after();
                const uint32_t scol = tmem + lane_addr + sb * 128;
                // pass 1: row maximum of the unmasked scores (four independent chains); on the
                // diagonal tile key c of the tile is visible to row r when c <= r
                float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    float v[32];
                    tmem_ld32(scol + c4 * 32, v);
                    if (!diag) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) mq[i & 3] = fmaxf(mq[i & 3], v[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (c4 * 32 + i <= r) mq[i & 3] = fmaxf(mq[i & 3], v[i]);
                    }
                }
                const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * a.scale_log2;
                const bool need = mx > m + LAZY;
                if (__any_sync(0xffffffffu, need)) {
                    const float nm = need ? softmax_max_update(m, mx) : m;
                    const float cf = softmax_rescale(m, nm);
                    if (j > 0) {
                        // the previous key tile's P V must have landed in O before it is rescaled
                        if (!wait_warp(&pv_done[(x - 1) & 1u], ((x - 1) >> 1) & 1u, abort_flag, a.status, lane)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int c2 = 0; c2 < 8; ++c2) {
                            float o[16];
                            tmem_ld16(tmem + lane_addr + O_COL + c2 * 16, o);
#pragma unroll
                            for (int i = 0; i < 16; ++i) o[i] *= cf;
                            tmem_st16(tmem + lane_addr + O_COL + c2 * 16, o);
                        }
                    }
                    l *= cf;
                    m = nm;
                }
                // the P buffer is free once the P V that read it two key tiles ago has completed
                if (x >= 2 && !wait_warp(&pv_done[pb], ((x - 2) >> 1) & 1u, abort_flag, a.status, lane)) {
                    ok = false;
                    break;
                }
                // pass 2: P = 2^(s * scale - m) (0 where masked) as bf16 into the P buffer, row r;
                // one FFMA and one ex2.approx per score, four partial row sums
                uint8_t* prow = smem + OFF_P + pb * TILE + r * 128;
                const float sl = a.scale_log2, negm = -m;
                float lq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    float v[32];
                    tmem_ld32(scol + c4 * 32, v);
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float p0 = ex2_approx(fmaf(v[2 * i], sl, negm));
                        float p1 = ex2_approx(fmaf(v[2 * i + 1], sl, negm));
                        if (diag) {
                            p0 = (c4 * 32 + 2 * i <= r) ? p0 : 0.f;
                            p1 = (c4 * 32 + 2 * i + 1 <= r) ? p1 : 0.f;
                        }
                        lq[i & 3] += p0 + p1;
                        pk[i] = pack_bf16x2(p0, p1);
                    }
                    uint8_t* hrow = prow + (c4 >> 1) * HALF_TILE;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int c = (c4 & 1) * 4 + q4;
                        *reinterpret_cast<uint4*>(hrow + ((c ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                    }
                }
                l += (lq[0] + lq[1]) + (lq[2] + lq[3]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sb]);
                if ((j + 1) * KEYS > C) {
                    // keys past the chunk in this tile: zero their V rows (after the copies landed)
                    if (!wait_warp(&v_full[st], (x / NS) & 1u, abort_flag, a.status, lane)) { ok = false; break; }
                    if (j * KEYS + r >= C) {
                        uint8_t* vrow = smem + OFF_V + st * TILE + r * 128;
#pragma unroll
                        for (int bb = 0; bb < 2; ++bb)
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                reinterpret_cast<uint4*>(vrow + bb * HALF_TILE)[c] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[pb]);
            }
            if (!ok) break;
            // ---- output row: O / l
            const uint32_t last = kt + qt;
            if (!wait_warp(&pv_done[last & 1u], (last >> 1) & 1u, abort_flag, a.status, lane)) { ok = false; break; }
            tc_fence_after();
            const float inv = 1.f / l;
            uint16_t* orow = a.out + ((size_t)(R + pos) * nq + h) * 128;
#pragma unroll
            for (int c2 = 0; c2 < 8; ++c2) {
                float o[16];
                tmem_ld16(tmem + lane_addr + O_COL + c2 * 16, o);
                if (pos < C) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(o[2 * i] * inv, o[2 * i + 1] * inv);
                    reinterpret_cast<uint4*>(orow + c2 * 16)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    reinterpret_cast<uint4*>(orow + c2 * 16)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
            kt += qt + 1;
        }
    }

    __syncthreads();
    if (threadIdx.x == 0)
        for (int i = 0; i < BARRIERS; ++i) mbar_inval(bars + i);
}

}  // namespace prefill_impl
}  // namespace nf
