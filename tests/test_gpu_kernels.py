"""Single-kernel parity on the GPU, through the C ABI.

GEMM: integer-valued bf16 operands make every fp32 accumulation exact, so the tcgen05
result must equal the integer matmul bit for bit (a wrong descriptor, swizzle, tile
index or k step shows up as a wrong number); random operands are checked against
float64. Attention: decode (with split-KV merge) and prefill against the float64 oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from synth import weights as SW
from synth.workloads import ModelShape, Workload

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def nf():
    import intra_device_overlapped_b200 as m
    return m


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(DEV).to(torch.bfloat16)


# --- generator -------------------------------------------------------------------------------------

@pytest.mark.parametrize("seed,tid,n,sigma,mean,offset", [
    (0, 7, 100_003, 0.02, 0.0, 0), (1, 3, 65_536, 1.0, 0.0, 12345), (0, 8, 4096, 0.1, 1.0, 0),
    (2, 0, 999, 1.0, 0.0, (1 << 32) + 5)])
def test_device_generator_matches_host(seed, tid, n, sigma, mean, offset):
    t = torch.empty(n, dtype=torch.bfloat16, device=DEV)
    synth.gpu_fill_normal_bf16(t.data_ptr(), n, seed, tid, sigma, mean, offset)
    torch.cuda.synchronize()
    got = t.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, synth.normal_bf16(seed, tid, n, sigma, mean, offset))


# --- GEMM ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(300, 512, 320), (1, 256, 64), (129, 768, 128), (1536, 1024, 4096)])
def test_gemm_integer_operands_bit_exact(nf, M, N, K):
    rng = np.random.default_rng(M * 7 + N)
    A = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
    B = rng.integers(-4, 5, size=(N, K)).astype(np.float32)
    ref = (A.astype(np.int64) @ B.astype(np.int64).T).astype(np.float32)
    a, b = _bf16(A), _bf16(B)
    for sms in (0, 1, 7):
        c = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
        nf.check(nf.nf_op_gemm_bf16(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, sms), "gemm")
        torch.cuda.synchronize()
        assert np.array_equal(c.cpu().numpy(), ref), f"sm_count={sms}"


def test_gemm_random_operands_vs_float64(nf):
    M, N, K = 777, 1280, 2048
    rng = np.random.default_rng(5)
    a = _bf16(rng.standard_normal((M, K)))
    b = _bf16(rng.standard_normal((N, K)) * 0.02)
    c = torch.empty((M, N), dtype=torch.float32, device=DEV)
    nf.check(nf.nf_op_gemm_bf16(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, 0), "gemm")
    torch.cuda.synchronize()
    ref = a.double().cpu().numpy() @ b.double().cpu().numpy().T
    err = np.abs(c.cpu().numpy() - ref).max()
    assert err < 1e-4 * np.abs(ref).max() + 1e-5


def test_gemm_rejects_bad_shapes(nf):
    a = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    c = torch.zeros((4, 256), dtype=torch.float32, device=DEV)
    assert nf.nf_op_gemm_bf16(a.data_ptr(), a.data_ptr(), c.data_ptr(), 4, 200, 64, 0) == nf.NF_ERR_INVALID_ARGUMENT
    assert nf.nf_op_gemm_bf16(a.data_ptr(), a.data_ptr(), c.data_ptr(), 4, 256, 60, 0) == nf.NF_ERR_INVALID_ARGUMENT


# --- attention -------------------------------------------------------------------------------------

ATT_SHAPES = {
    # d = 128, G = 4; contexts long enough for two KV splits; ragged chunk (not a multiple of 16 or 64)
    "d128": Workload(ModelShape("attn128", 1, 1024, 8, 2, 128, 512), 24, 1, 900, prefill_len=100),
    # d = 64, G = 2 (the tiny model's heads)
    "d64": Workload(ModelShape("attn64", 1, 256, 4, 2, 64, 512), 9, 0, 70, prefill_len=45),
    # G = 8 (Llama-2-70B head grouping)
    "g8": Workload(ModelShape("attn_g8", 1, 2048, 16, 2, 128, 512), 5, 300, 600, prefill_len=17),
    # 8 KV heads x 128, 32 / 64 query heads: the tensor-core decode kernel (whole pages, all heads)
    "tc32": Workload(ModelShape("attn_tc32", 1, 1024, 32, 8, 128, 512), 40, 0, 700, prefill_len=100),
    "tc64": Workload(ModelShape("attn_tc64", 1, 1024, 64, 8, 128, 512), 13, 200, 1100, prefill_len=33),
}


@pytest.fixture(scope="module", params=sorted(ATT_SHAPES))
def att_case(request, nf):
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = ATT_SHAPES[request.param]
    dw = DeviceWorkload(w, DEV)
    s = w.shape
    rng = np.random.default_rng(11)
    q = _bf16(rng.standard_normal((dw.T, s.n_q_heads, s.head_dim)))
    yield dw, q
    dw.close()


# Attention outputs (bf16) are compared with the absolute bar of the parity tests, 2e-2, against
# both readings of the oracle's attention: the bf16 model (P = bf16 weights) and exact float64.
ATT_ABS = 2e-2


def _att_excess(got, q, K, V, decode=True):
    """Largest |got - ref| over both readings (decode: one query [nq, d]; else a causal chunk)."""
    from oracle import forward as F
    worst = 0.0
    for bf in (True, False):
        ref = F.decode_attention(q, K, V, bf16_p=bf) if decode else F.prefill_attention(q, K, V, bf16_p=bf)
        worst = max(worst, float(np.max(np.abs(got - ref))) if ref.size else 0.0)
    return worst


def _oracle_kv(dw, r):
    from oracle import forward as F
    b, s = dw.batch, dw.shape
    pages = b.page_indices[b.page_indptr[r]:b.page_indptr[r + 1]]
    kv = F.PagedKV(lambda layer, pg: synth.bf16_to_f64(SW.host_kv_pages(s, layer, pg)), s.page_size)
    return kv, pages


def test_decode_attention_vs_oracle(nf, att_case):
    from oracle import forward as F
    dw, q = att_case
    b = dw.batch
    out = torch.zeros_like(q)
    nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), out.data_ptr(), dw.io, 0, 0, b.num_decode, 0), "dec")
    nf.check(dw.sync(), "status")
    qd = q.double().cpu().numpy()
    got = out.float().cpu().numpy()
    worst = 0.0
    for r in range(b.num_decode):
        kv, pages = _oracle_kv(dw, r)
        K, V = kv.read(0, pages, int(b.ctx_lens[r]) + 1)
        worst = max(worst, _att_excess(got[r], qd[r], K, V))
    print(f"decode attention, {b.num_decode} requests: max-abs {worst:.4g}")
    assert worst <= ATT_ABS, worst


def test_decode_attention_independent_of_grouping_and_grid(nf, att_case):
    dw, q = att_case
    R = dw.batch.num_decode
    full = torch.zeros_like(q)
    nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), full.data_ptr(), dw.io, 0, 0, R, 0), "dec")
    part = torch.zeros_like(q)
    cut = R // 3
    nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), part.data_ptr(), dw.io, 0, 0, cut, 5), "dec")
    nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), part.data_ptr(), dw.io, 0, cut, R, 17), "dec")
    nf.check(dw.sync(), "status")
    assert torch.equal(full[:R].view(torch.int16), part[:R].view(torch.int16))


def test_prefill_attention_vs_oracle(nf, att_case):
    from oracle import forward as F
    dw, q = att_case
    b = dw.batch
    R, C = b.num_decode, b.prefill_len
    out = torch.zeros_like(q)
    nf.check(nf.nf_op_prefill_attention(dw.model, q.data_ptr(), out.data_ptr(), dw.io, 0, R, C, 0), "pre")
    nf.check(dw.sync(), "status")
    kv, pages = _oracle_kv(dw, R)
    K, V = kv.read(0, pages, C)
    got = out.float().cpu().numpy()[R:R + C]
    err = _att_excess(got, q.double().cpu().numpy()[R:R + C], K, V, decode=False)
    print(f"prefill attention, {C} rows: max-abs {err:.4g}")
    assert err <= ATT_ABS
    # grid size does not change the result
    out2 = torch.zeros_like(q)
    nf.check(nf.nf_op_prefill_attention(dw.model, q.data_ptr(), out2.data_ptr(), dw.io, 0, R, C, 3), "pre")
    nf.check(dw.sync(), "status")
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


# --- bounded device waits --------------------------------------------------------------------------

def test_device_wait_times_out_cleanly(nf):
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert nf.nf_op_wait_flag_test(flag.data_ptr(), 10_000_000) == nf.NF_ERR_DEVICE_TIMEOUT
    flag.fill_(1)
    torch.cuda.synchronize()
    assert nf.nf_op_wait_flag_test(flag.data_ptr(), 10_000_000) == nf.NF_OK
    # the context is still healthy: a GEMM runs and is exact
    a = torch.ones((128, 64), dtype=torch.bfloat16, device=DEV)
    c = torch.zeros((128, 256), dtype=torch.float32, device=DEV)
    b = torch.ones((256, 64), dtype=torch.bfloat16, device=DEV)
    nf.check(nf.nf_op_gemm_bf16(a.data_ptr(), b.data_ptr(), c.data_ptr(), 128, 256, 64, 0), "gemm")
    torch.cuda.synchronize()
    assert torch.all(c == 64.0)


def test_tc64_decode_many_request_ends_per_cta_is_deterministic(nf):
    """64 query heads (fewer V stages than P buffers), many short requests per CTA: repeated runs and
    every grid give the same bits, and rows match the oracle (regression for the last-page V rows)."""
    from oracle import forward as F
    from intra_device_overlapped_b200.harness import DeviceWorkload
    w = Workload(ModelShape("attn_tc64_many", 1, 1024, 64, 8, 128, 512), 160, 0, 120, prefill_len=16)
    dw = DeviceWorkload(w, DEV)
    try:
        rng = np.random.default_rng(19)
        q = _bf16(rng.standard_normal((dw.T, 64, 128)))
        R = dw.batch.num_decode
        outs = []
        for grid in (3, 3, 7, 0):
            out = torch.zeros_like(q)
            nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), out.data_ptr(), dw.io, 0, 0, R, grid), "dec")
            nf.check(dw.sync(), "status")
            outs.append(out[:R].view(torch.int16).clone())
        for o in outs[1:]:
            assert torch.equal(o, outs[0])
        got = outs[0].view(torch.bfloat16).float().cpu().numpy()
        qd = q.double().cpu().numpy()
        worst = 0.0
        for r in range(0, R, 7):
            kv, pages = _oracle_kv(dw, r)
            K, V = kv.read(0, pages, int(dw.batch.ctx_lens[r]) + 1)
            worst = max(worst, _att_excess(got[r], qd[r], K, V))
        assert worst <= ATT_ABS, worst
    finally:
        dw.close()


# --- decode attention edge cases: explicit context lengths ---------------------------------------------

# Contexts of 0 keys cached (the new key alone), one page minus one / exactly / plus one, the split
# boundary of the tensor-core kernel (chunks of at most 64 pages of 16 keys: 1023 / 1024 / 1025 keys)
# and the longest Mixtral context (4096 cached, 257 pages, 5 chunks).
EDGE_CTX = [0, 15, 16, 17, 31, 510, 511, 1022, 1023, 1024, 2047, 4096, 4095, 100, 1]


@pytest.mark.parametrize("nq", [32, 64])
def test_decode_attention_edge_contexts(nf, nq):
    from synth.workloads import batch_for_contexts
    from intra_device_overlapped_b200.harness import DeviceWorkload
    shape = ModelShape(f"attn_edge{nq}", 1, 1024, nq, 8, 128, 512)
    w = Workload(shape, len(EDGE_CTX), prefill_len=16)
    dw = DeviceWorkload(w, DEV, batch=batch_for_contexts(shape, EDGE_CTX, 16))
    try:
        rng = np.random.default_rng(23 + nq)
        q = _bf16(rng.standard_normal((dw.T, nq, 128)) * 2.0)   # sharper softmax: rescales happen
        R = dw.batch.num_decode
        outs = []
        for grid in (0, 1, 3, 7):
            out = torch.full_like(q, float("nan"))
            nf.check(nf.nf_op_decode_attention(dw.model, q.data_ptr(), out.data_ptr(), dw.io, 0, 0, R, grid), "dec")
            nf.check(dw.sync(), "status")
            outs.append(out[:R].view(torch.int16).clone())
        for o in outs[1:]:
            assert torch.equal(o, outs[0])          # the split depends on the context only, not on the grid
        got = outs[0].view(torch.bfloat16).float().cpu().numpy()
        qd = q.double().cpu().numpy()
        for r, c in enumerate(EDGE_CTX):
            kv, pages = _oracle_kv(dw, r)
            K, V = kv.read(0, pages, c + 1)
            err = _att_excess(got[r], qd[r], K, V)
            assert err <= ATT_ABS, (c, err)
    finally:
        dw.close()
