"""Model creation that fails part-way returns a status and leaves no device memory behind.

nf_init_model allocates its workspaces one after another; here the SwiGLU activation buffer
(max_tokens x ffn bf16, about 2 TB) cannot be allocated while the buffers before it can. The call must
return NF_ERR_OUT_OF_MEMORY with no model, and free what it had allocated: free device memory is the
same after three such calls as before them.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _cfg(nf, ffn):
    return nf.nf_model_config(n_layers=1, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=ffn, vocab=0,
                              n_experts=0, top_k=0, rms_eps=1e-5, rope_theta=10000.0, page_size=16,
                              max_tokens=1024, max_requests=8, max_position=512)


def test_failed_init_frees_its_device_memory():
    import intra_device_overlapped_b200 as nf
    torch.cuda.set_device(DEV)
    st, h = nf.nf_init_model(_cfg(nf, 512))            # a model that fits: warms up the context
    assert st == nf.NF_OK and h
    nf.nf_destroy_model(h)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        st, h = nf.nf_init_model(_cfg(nf, 1 << 30))
        assert st == nf.NF_ERR_OUT_OF_MEMORY and not h
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free0 - free1 < (8 << 20), (free0, free1)
