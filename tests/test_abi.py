"""The C ABI library loads, exports every declared entry point, and its host-only logic
(configuration validation, the planner) behaves as documented. CPU only."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nf():
    from intra_device_overlapped_b200 import build
    build.build()
    import intra_device_overlapped_b200 as m
    return m


def _declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(nf_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(nf):
    declared = _declared_symbols()
    assert len(declared) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", nf.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (nf_\w+)$", out, flags=re.M))
    assert declared <= exported, declared - exported
    lib = ctypes.CDLL(nf.LIB_PATH)
    for name in declared:
        assert getattr(lib, name) is not None
    assert set(nf.EXPORTED) == declared


def test_library_has_no_driver_dependency(nf):
    out = subprocess.run(["ldd", nf.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_status_strings(nf):
    for code in range(7):
        assert nf.nf_status_string(code) != "unknown status"
    assert nf.nf_status_string(99) == "unknown status"
    assert "sm_100a" in nf.nf_version()


def _cfg(nf, **kw):
    from intra_device_overlapped_b200.harness import model_config
    from synth.workloads import WORKLOADS
    c = model_config(WORKLOADS["tiny_layer"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_init_without_device_or_with_bad_config(nf):
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only check")
    st, h = nf.nf_init_model(_cfg(nf))
    assert st == nf.NF_ERR_CUDA and not h
    st, _ = nf.nf_init_model(_cfg(nf, page_size=32))
    assert st in (nf.NF_ERR_UNSUPPORTED, nf.NF_ERR_INVALID_ARGUMENT)
    st, _ = nf.nf_init_model(_cfg(nf, head_dim=96))
    assert st == nf.NF_ERR_UNSUPPORTED


def _desc(nf, b):
    ctx = np.ascontiguousarray(b.ctx_lens, dtype=np.int32)
    ip = np.ascontiguousarray(b.page_indptr, dtype=np.int32)
    pg = np.ascontiguousarray(b.page_indices, dtype=np.int32)
    d = nf.nf_batch_desc(num_decode=b.num_decode, prefill_len=b.prefill_len, prefix_len=0,
                         ctx_len=ctx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                         page_indptr=ip.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), num_pages=b.num_pages,
                         page_indices=pg.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    return d, (ctx, ip, pg)


@pytest.mark.parametrize("name", ["tiny_layer", "llama3_8b_layer", "llama3_8b_full", "llama2_70b_slice",
                                  "mixtral_8x7b_slice"])
def test_planner_produces_valid_plans(nf, name):
    from intra_device_overlapped_b200.harness import model_config
    from synth.workloads import WORKLOADS, make_batch
    w = WORKLOADS[name]
    b = make_batch(w)
    d, keep = _desc(nf, b)
    for opts in (nf.nf_plan_opts(force_template=-1), nf.nf_plan_opts(force_nano=2, force_template=1),
                 nf.nf_plan_opts(force_nano=4, force_template=1, force_sm_attn=40),
                 nf.nf_plan_opts(force_nano=1, force_template=0),
                 nf.nf_plan_opts(force_nano=1, force_template=2, force_sm_attn=124)):
        st, p = nf.nf_plan_for_config(model_config(w), 148, d, opts)
        assert st == 0
        T = b.num_tokens
        assert p.num_tokens == T and p.tok_begin[0] == 0 and p.tok_end[p.n_nano - 1] == T
        for j in range(p.n_nano - 1):
            assert p.tok_end[j] == p.tok_begin[j + 1]
        for j in range(p.n_nano):
            assert p.tok_end[j] > p.tok_begin[j]
            assert not (b.num_decode < p.tok_begin[j] < T)       # the chunk is never split
        assert sorted(p.nano_order[i] for i in range(p.n_nano)) == list(range(p.n_nano))
        if p.order_template != nf.NF_TEMPLATE_SEQUENTIAL:
            assert p.sm_attn + p.sm_gemm <= 148 and p.sm_attn >= 1
            assert p.predicted_us <= p.predicted_serial_us * 1.2
        if opts.force_nano:
            assert p.n_nano == opts.force_nano
        if opts.force_sm_attn:
            assert p.sm_attn == opts.force_sm_attn
    assert p.kv_pages_read > 0


def test_planner_rejects_short_page_table(nf):
    from intra_device_overlapped_b200.harness import model_config
    from synth.workloads import WORKLOADS, make_batch
    w = WORKLOADS["tiny_layer"]
    b = make_batch(w)
    b.page_indptr = b.page_indptr.copy()
    b.page_indptr[1:] -= 1          # request 0 loses a page
    d, keep = _desc(nf, b)
    st, _ = nf.nf_plan_for_config(model_config(w), 148, d, None)
    assert st == nf.NF_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("bad", [-1, "num_pages", "missing"])
def test_planner_rejects_page_ids_outside_the_pool(nf, bad):
    """A page id < 0 or >= num_pages anywhere in the host page table (or no host table at all) is
    rejected on the host with NF_ERR_INVALID_ARGUMENT, before any launch."""
    from intra_device_overlapped_b200.harness import model_config
    from synth.workloads import WORKLOADS, make_batch
    w = WORKLOADS["tiny_layer"]
    b = make_batch(w)
    d, keep = _desc(nf, b)
    st, _ = nf.nf_plan_for_config(model_config(w), 148, d, None)
    assert st == 0
    pg = keep[2]
    if bad == "missing":
        d.page_indices = ctypes.POINTER(ctypes.c_int32)()
    else:
        pg[int(b.page_indptr[3]) + 1] = -1 if bad == -1 else b.num_pages   # one id of request 3
    st, _ = nf.nf_plan_for_config(model_config(w), 148, d, None)
    assert st == nf.NF_ERR_INVALID_ARGUMENT


def test_planner_prefers_overlap_on_the_8b_layer(nf):
    from intra_device_overlapped_b200.harness import model_config
    from synth.workloads import WORKLOADS, make_batch
    w = WORKLOADS["llama3_8b_layer"]
    b = make_batch(w)
    d, keep = _desc(nf, b)
    st, p = nf.nf_plan_for_config(model_config(w), 148, d, None)
    assert st == 0 and p.order_template != nf.NF_TEMPLATE_SEQUENTIAL and p.n_nano >= 2
    st, seq = nf.nf_plan_for_config(model_config(w), 148, d, nf.nf_plan_opts(force_nano=1, force_template=0))
    assert p.predicted_us < seq.predicted_us


def test_planner_fuzz_returns_valid_plans_or_invalid_argument(nf):
    """Random batches (including empty decode sets, no prefill, tiny and long contexts, short page
    tables) and random forced options: every call returns a plan that covers the batch with the
    chunk whole, or NF_ERR_INVALID_ARGUMENT; none crashes."""
    from intra_device_overlapped_b200.harness import model_config
    from synth.workloads import WORKLOADS
    rng = np.random.default_rng(99)
    cfg = model_config(WORKLOADS["llama3_8b_layer"])
    ok = 0
    for case in range(300):
        R = int(rng.choice([0, 1, 2, 7, 64, 300]))
        C = int(rng.choice([0, 1, 17, 128, 1000]))
        if R + C == 0:
            continue
        ctx = rng.integers(0, 3000, R).astype(np.int32)
        counts = [(int(c) + 1 + 15) // 16 for c in ctx] + [(C + 15) // 16]
        if rng.random() < 0.1 and R:
            counts[int(rng.integers(0, R))] -= 1  # one request short of a page: must be rejected
        indptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        pages = rng.permutation(max(int(indptr[-1]), 1)).astype(np.int32)
        d = nf.nf_batch_desc(num_decode=R, prefill_len=C, prefix_len=0,
                             ctx_len=ctx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                             page_indptr=indptr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                             num_pages=max(int(indptr[-1]), 1),
                             page_indices=pages.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
        opts = nf.nf_plan_opts(force_nano=int(rng.integers(0, 5)), force_sm_attn=int(rng.choice([0, 8, 64, 140])),
                               force_template=int(rng.integers(-1, 3)))
        if opts.force_nano == 0 and opts.force_template == -1:
            opts.force_nano = 1  # keep the full search (milliseconds per call) out of the loop
        st, p = nf.nf_plan_for_config(cfg, 148, d, opts)
        assert st in (0, nf.NF_ERR_INVALID_ARGUMENT), (case, st)
        short = any(c < ((int(x) + 1 + 15) // 16) for c, x in zip(counts[:R], ctx))
        if short:
            assert st == nf.NF_ERR_INVALID_ARGUMENT, case
        if st != 0:
            continue
        ok += 1
        T = R + C
        assert p.num_tokens == T and p.tok_begin[0] == 0 and p.tok_end[p.n_nano - 1] == T
        for j in range(p.n_nano):
            assert p.tok_end[j] > p.tok_begin[j]
            assert not (R < p.tok_begin[j] < T)
        assert sorted(p.nano_order[i] for i in range(p.n_nano)) == list(range(p.n_nano))
        if p.order_template != nf.NF_TEMPLATE_SEQUENTIAL:
            assert 1 <= p.sm_attn and p.sm_attn + p.sm_gemm <= 148
    assert ok > 100


def test_offload_rejects_bad_arguments_without_a_device(nf):
    """nf_offload_kv validates on the host: a null model, empty page list or empty layer range is
    rejected before anything is launched."""
    import ctypes
    pools = (ctypes.c_void_p * 1)(None)
    buf = ctypes.create_string_buffer(16)
    assert nf.nf_offload_kv(None, pools, 4, [0, 1], 0, 1, ctypes.addressof(buf), 0) == nf.NF_ERR_INVALID_ARGUMENT
    assert nf.nf_offload_kv(None, pools, 4, [], 0, 1, ctypes.addressof(buf), 0) == nf.NF_ERR_INVALID_ARGUMENT
