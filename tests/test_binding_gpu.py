"""The Python binding refuses caller-provided outputs and workspaces that do
not match the call (shape, dtype, device) before anything is launched, and
accepts the matching ones."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from sparse_long_context_nsa_b200 import _build
    _build.build()
    import sparse_long_context_nsa_b200 as m
    return m


def _inputs(S=512, n1=8, n2=2, dd=64, l=32, d=16, lp=64):
    g = torch.Generator().manual_seed(3)
    q = torch.randn(S, n1, dd, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(S, n2, dd, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(S, n2, dd, generator=g).to(torch.bfloat16).cuda()
    w = (torch.rand(l, n2, generator=g) * 2 / l).to(torch.bfloat16).cuda()
    return q, k, v, w


def test_compress_checks_preallocated_outputs(nsa):
    q, k, v, w = _inputs()
    cuc = nsa.nsa_compress_out_len([512], 32, 16)
    tc = int(cuc[-1])
    good = torch.empty(tc, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="kcmp"):
        nsa.nsa_compress(k, v, w, 32, 16, [512], kcmp=torch.empty(tc - 1, 2, 64, dtype=torch.bfloat16, device="cuda"),
                         vcmp=good.clone())
    with pytest.raises(ValueError, match="vcmp"):
        nsa.nsa_compress(k, v, w, 32, 16, [512], kcmp=good.clone(),
                         vcmp=torch.empty(tc, 2, 64, dtype=torch.float16, device="cuda"))
    kc, vc = nsa.nsa_compress(k, v, w, 32, 16, [512], kcmp=good.clone(), vcmp=good.clone())
    assert kc.shape == (tc, 2, 64) and nsa.nsa_compress_status() == 0


def test_attention_checks_outputs_workspace_and_masks(nsa):
    q, k, v, w = _inputs()
    cuc = nsa.nsa_compress_out_len([512], 32, 16)
    kc, vc = nsa.nsa_compress(k, v, w, 32, 16, [512])
    args = (q, kc, vc, 0.125, 8, 32, 16, 64, 4, [512], cuc, [8])
    att = torch.empty(512, 8, 64, dtype=torch.bfloat16, device="cuda")
    tk = torch.empty(512, 2, 4, dtype=torch.int32, device="cuda")
    st = torch.empty(512, 8, 8, dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError, match="topk_indices"):
        nsa.nsa_compress_attention(*args, out=(att, tk[:, :, :3].contiguous(), st, st.clone()))
    with pytest.raises(ValueError, match="softmax_max"):
        nsa.nsa_compress_attention(*args, out=(att, tk, st.half(), st.clone()))
    with pytest.raises(ValueError, match="workspace"):
        nsa.nsa_compress_attention(*args, workspace=torch.empty(1 << 20, dtype=torch.float32, device="cuda"))
    # an undersized workspace is refused, never silently replaced: the kernel's
    # error word must land in the tensor the caller reads it back from
    need = nsa.nsa_compress_attention_workspace_size(8, 2, 64, 64, 32, 16, 64, 4, [512], cuc, [8])
    small = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError, match="workspace"):
        nsa.nsa_compress_attention(*args, workspace=small)
    sneed = nsa.nsa_select_attention_workspace_size(8, 2, 64, 64, 64, 4, [512], [512])
    tk0 = torch.zeros(512, 2, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError, match="workspace"):
        nsa.nsa_select_attention(q, k, v, tk0, 0.125, 8, 64, [512], [512],
                                 workspace=torch.zeros(sneed - 1, dtype=torch.uint8, device="cuda"))
    with pytest.raises(TypeError, match="atten_mask"):
        nsa.nsa_compress_attention(*args, atten_mask=torch.zeros(512, 64, dtype=torch.float32, device="cuda"))
    res = nsa.nsa_compress_attention(*args, out=(att, tk, st, st.clone()))
    assert res[0] is att and int(res[1].min()) >= -1
    res = nsa.nsa_compress_attention_noalloc(*args, out=(att, tk, st, st.clone()))
    with pytest.raises(ValueError, match="attention_out"):
        nsa.nsa_compress_attention_noalloc(*args, out=(att[:500], tk, st, st.clone()))


def test_select_checks_outputs(nsa):
    q, k, v, w = _inputs()
    tk = torch.full((512, 2, 4), -1, dtype=torch.int32, device="cuda")
    tk[:, :, 0] = 0
    att = torch.empty(512, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="softmax_lse"):
        nsa.nsa_select_attention(q, k, v, tk, 0.125, 8, 64, [512], [512],
                                 out=(att, torch.empty(512, 8, 1, device="cuda")))
    out, lse = nsa.nsa_select_attention(q, k, v, tk, 0.125, 8, 64, [512], [512],
                                        out=(att, torch.empty(512, 8, device="cuda")))
    assert out is att and torch.isfinite(lse).all()
