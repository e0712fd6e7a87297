"""Host-only checks of the C ABI (no GPU needed): the library loads, exports
every function include/kda.h declares, and rejects bad arguments before
enqueuing anything."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_124_b200 as kda
from gated_delta_rule_124_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_binding_exports():
    assert sorted(kda.EXPORTS) == declared_functions()


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for code in range(7):
        s = kda.status_string(code)
        assert s.startswith("KDA_"), s
    assert "UNKNOWN" in kda.status_string(99)


def test_workspace_size_rules(lib):
    f = kda.kda_chunk_fwd_workspace_size
    assert f(4096, 2, 32, 128, 128, 64, "bf16") > 0
    assert f(64, 1, 1, 32, 32, 16, "f32") > 0
    assert f(64, 1, 1, 48, 32, 16, "f32") == 0   # unsupported dk
    assert f(64, 1, 1, 32, 32, 8, "f32") == 0    # unsupported chunk
    assert f(64, 0, 1, 32, 32, 16, "f32") == 0   # no sequences
    # grows with tokens
    assert f(8192, 2, 32, 64, 64, 64, "f32") > f(4096, 2, 32, 64, 64, 64, "f32")


def test_chunk_upper_bound(lib):
    assert kda.kda_num_chunks_upper_bound(4096, 2, 64) == 64 + 1  # (4096 + 2*63) // 64
    assert kda.kda_num_chunks_upper_bound(0, 3, 16) == 2
    # bound covers any split of 100 tokens into 3 sequences
    for a in range(0, 101, 7):
        for b in range(0, 101 - a, 11):
            c = 100 - a - b
            used = sum((x + 15) // 16 for x in (a, b, c))
            assert used <= kda.kda_num_chunks_upper_bound(100, 3, 16)


FAKE = 1 << 20  # a 16-byte-aligned non-NULL address; never dereferenced on these paths


def _fwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, initial_state=None, cu_seqlens=None,
                B=1, T=64, num_seqs=1, H=1, dk=32, dv=32, chunk=16, dtype="f32", o=FAKE,
                final_state=None, workspace=FAKE * 2, workspace_bytes=1 << 40, stream=0,
                check=False)
    args.update(kw)
    return kda.kda_chunk_fwd(**args)


def test_chunk_fwd_rejects_bad_arguments(lib):
    assert _fwd(q=None) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(o=None) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(k=FAKE + 4) == kda.KDA_ERR_INVALID_ARG          # misaligned
    assert _fwd(B=0) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(T=-1) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(num_seqs=2) == kda.KDA_ERR_INVALID_ARG          # != B without cu_seqlens
    assert _fwd(cu_seqlens=FAKE, B=2, num_seqs=2) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(dk=48) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(chunk=128) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(dtype=kda.KDA_DTYPE_F32, workspace=None) == kda.KDA_ERR_WORKSPACE
    assert _fwd(workspace_bytes=16) == kda.KDA_ERR_WORKSPACE
    assert _fwd(workspace=FAKE + 16) == kda.KDA_ERR_INVALID_ARG  # not 256-aligned
    assert _fwd(final_state=FAKE + 8) == kda.KDA_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(lib):
    def dec(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, state=FAKE, o=FAKE, N=4, H=2,
                 dk=128, dv=128, dtype="bf16", stream=0, check=False)
        a.update(kw)
        return kda.kda_decode_step(**a)
    assert dec(state=None) == kda.KDA_ERR_INVALID_ARG
    assert dec(q=FAKE + 2) == kda.KDA_ERR_INVALID_ARG
    assert dec(N=-1) == kda.KDA_ERR_INVALID_ARG
    assert dec(H=0) == kda.KDA_ERR_INVALID_ARG
    assert dec(dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert dec(N=0) == kda.KDA_OK                                 # nothing to do
    assert dec(N=0, q=None) == kda.KDA_OK


def test_step_calls_reject_bad_arguments(lib):
    common = dict(cu_seqlens=None, B=1, T=64, num_seqs=1, H=1, chunk=16, workspace=FAKE * 2,
                  workspace_bytes=1 << 40, stream=0, check=False)
    assert kda.kda_chunk_gate_cumsum(g=None, dk=32, G=FAKE, **common) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_intra(k=FAKE, v=FAKE, G=FAKE, beta=FAKE, dk=32, dv=32, dtype="f32",
                               W=None, Ut=FAKE, **common) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_inter(k=FAKE, G=FAKE, W=FAKE, U=FAKE, initial_state=FAKE + 4, dk=32,
                               dv=32, dtype="f32", chunk_states=FAKE, final_state=None,
                               **common) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_output(q=FAKE, k=FAKE, G=FAKE, U=FAKE, chunk_states=FAKE, dk=32,
                                dv=96, dtype="f32", o=FAKE, **common) == kda.KDA_ERR_UNSUPPORTED


def test_plan_query(lib):
    f = kda.kda_chunk_fwd_plan
    assert f(4096, 2, 32, 128, 128, 64, "bf16") in (kda.KDA_PLAN_SIMT, kda.KDA_PLAN_SPLIT,
                                                   kda.KDA_PLAN_OVERLAP)
    assert f(64, 1, 1, 32, 32, 16, "f32") == kda.KDA_PLAN_SIMT   # no tensor-core plan
    assert f(64, 3, 1, 32, 32, 16, "f32", packed=True) == kda.KDA_PLAN_SIMT
    assert f(64, 1, 1, 48, 32, 16, "f32") == -1
    assert f(64, 0, 1, 32, 32, 16, "f32") == -1
    assert f(-1, 1, 1, 32, 32, 16, "f32") == -1


def test_split_calls_reject_bad_arguments(lib):
    f = kda.kda_chunk_split_workspace_size
    assert f(4096, 2, 32) > 0
    assert f(8192, 2, 32) > f(4096, 2, 32)
    assert f(4096, 0, 32) == 0 and f(-1, 1, 32) == 0 and f(64, 1, 0) == 0
    common = dict(cu_seqlens=None, B=1, T=64, num_seqs=1, H=1, workspace=FAKE * 2,
                  workspace_bytes=1 << 40, stream=0, check=False)
    intra = dict(q=FAKE, k=FAKE, g=FAKE, beta=FAKE, **common)
    chain = dict(v=FAKE, initial_state=None, o=FAKE, final_state=None, **common)
    assert kda.kda_chunk_split_intra(**{**intra, "q": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_split_intra(**{**intra, "g": FAKE + 4}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_split_intra(**{**intra, "B": 0}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_split_intra(**{**intra, "num_seqs": 2}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_split_chain(**{**chain, "o": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_split_chain(**{**chain, "v": FAKE + 2}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_split_chain(**{**chain, "H": 0}) == kda.KDA_ERR_INVALID_ARG


def test_get_device_status_rejects_bad_workspace(lib):
    assert kda.kda_get_device_status(None, 0) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_get_device_status(FAKE + 16, 0) == kda.KDA_ERR_INVALID_ARG


def test_layer_calls_reject_bad_arguments(lib):
    conv = dict(xq=FAKE, xk=FAKE, xv=FAKE, wq=FAKE, wk=FAKE, wv=FAKE, cu_seqlens=None, B=1,
                T=64, num_seqs=1, H=2, dk=128, dv=128, dtype="bf16", eps=1e-6, q=FAKE, k=FAKE,
                v=FAKE, stream=0, check=False)
    assert kda.kda_qkv_conv_norm(**{**conv, "xq": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm(**{**conv, "wk": FAKE + 4}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm(**{**conv, "eps": 0.0}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm(**{**conv, "eps": float("nan")}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm(**{**conv, "dk": 96}) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_qkv_conv_norm(**{**conv, "num_seqs": 2}) == kda.KDA_ERR_INVALID_ARG
    gate = dict(o=FAKE, gate=FAKE, w=FAKE, total_tokens=64, H=2, dv=64, dtype="f32", eps=1e-6,
                y=FAKE, stream=0, check=False)
    assert kda.kda_output_norm_gate(**{**gate, "y": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_output_norm_gate(**{**gate, "total_tokens": -1}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_output_norm_gate(**{**gate, "dv": 48}) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_output_norm_gate(**{**gate, "eps": -1.0}) == kda.KDA_ERR_INVALID_ARG


def test_gdn_calls_reject_bad_arguments(lib):
    f = kda.kda_gdn_chunk_fwd_workspace_size
    assert f(4096, 2, 32, 128, 128, 64, "bf16") >= kda.kda_chunk_fwd_workspace_size(
        4096, 2, 32, 128, 128, 64, "bf16")
    assert f(64, 1, 1, 48, 32, 16, "f32") == 0
    args = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, initial_state=None, cu_seqlens=None,
                B=1, T=64, num_seqs=1, H=1, dk=32, dv=32, chunk=16, dtype="f32", o=FAKE,
                final_state=None, workspace=FAKE * 2, workspace_bytes=16, stream=0, check=False)
    assert kda.kda_gdn_chunk_fwd(**{**args, "g": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_gdn_chunk_fwd(**{**args, "beta": FAKE + 4}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_gdn_chunk_fwd(**{**args, "dk": 96}) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_gdn_chunk_fwd(**args) == kda.KDA_ERR_WORKSPACE       # 16 bytes
    dec = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, state=FAKE, o=FAKE, N=2, H=2, dk=128,
               dv=128, dtype="bf16", stream=0, check=False)
    assert kda.kda_gdn_decode_step(**{**dec, "state": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_gdn_decode_step(**{**dec, "dv": 40}) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_gdn_decode_step(**{**dec, "N": 0}) == kda.KDA_OK


def test_backward_call_rejects_bad_arguments(lib):
    assert kda.kda_chunk_bwd_workspace_size(4096, 2, 32, 128, 128) > 0
    assert kda.kda_chunk_bwd_workspace_size(4096, 2, 32, 96, 128) == 0
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, initial_state=None, dout=FAKE,
             dfinal_state=None, cu_seqlens=None, B=1, T=64, num_seqs=1, H=1, dk=32, dv=32,
             dtype="f32", dq=FAKE, dk_out=FAKE, dv_out=FAKE, dg=FAKE, dbeta=FAKE,
             dinitial_state=None, workspace=FAKE * 2, workspace_bytes=16, stream=0, check=False)
    assert kda.kda_chunk_bwd(**{**a, "dout": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_bwd(**{**a, "dg": FAKE + 4}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_bwd(**{**a, "dinitial_state": FAKE + 8}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_chunk_bwd(**{**a, "dk": 48}) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_chunk_bwd(**a) == kda.KDA_ERR_WORKSPACE


def test_gdn_backward_call_rejects_bad_arguments(lib):
    n = kda.kda_chunk_bwd_workspace_size(4096, 2, 32, 128, 128)
    m = kda.kda_gdn_chunk_bwd_workspace_size(4096, 2, 32, 128, 128)
    assert m >= n + 2 * 4096 * 32 * 128 * 4  # the spread gate and its gradient
    assert kda.kda_gdn_chunk_bwd_workspace_size(4096, 2, 32, 128, 40) == 0
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, initial_state=None, dout=FAKE,
             dfinal_state=None, cu_seqlens=None, B=1, T=64, num_seqs=1, H=1, dk=32, dv=32,
             dtype="f32", dq=FAKE, dk_out=FAKE, dv_out=FAKE, dg=FAKE, dbeta=FAKE,
             dinitial_state=None, workspace=FAKE * 2, workspace_bytes=16, stream=0, check=False)
    assert kda.kda_gdn_chunk_bwd(**{**a, "g": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_gdn_chunk_bwd(**{**a, "dg": FAKE + 4}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_gdn_chunk_bwd(**{**a, "dv": 40}) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_gdn_chunk_bwd(**{**a, "num_seqs": 2}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_gdn_chunk_bwd(**a) == kda.KDA_ERR_WORKSPACE


def test_conv_step_rejects_bad_arguments(lib):
    a = dict(xq=FAKE, xk=FAKE, xv=FAKE, wq=FAKE, wk=FAKE, wv=FAKE, conv_q=FAKE, conv_k=FAKE,
             conv_v=FAKE, N=4, H=2, dk=128, dv=128, dtype="bf16", eps=1e-6, q=FAKE, k=FAKE,
             v=FAKE, stream=0, check=False)
    assert kda.kda_qkv_conv_norm_step(**{**a, "conv_k": None}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm_step(**{**a, "xv": FAKE + 2}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm_step(**{**a, "dk": 96}) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_qkv_conv_norm_step(**{**a, "eps": 0.0}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm_step(**{**a, "N": -1}) == kda.KDA_ERR_INVALID_ARG
    assert kda.kda_qkv_conv_norm_step(**{**a, "N": 0}) == kda.KDA_OK


def test_explicit_plan_rules(lib):
    """kda_chunk_fwd_with_plan: an unknown plan is an invalid argument; a
    plan's workspace size is 0 where it cannot run (a tensor-core plan for
    fp32, or for another head dimension)."""
    ws = kda.kda_chunk_fwd_plan_workspace_size
    assert ws("simt", 4096, 2, 32, 128, 128, 64, "bf16") > 0
    assert ws("split", 4096, 2, 32, 128, 128, 64, "f32") == 0
    assert ws("split", 4096, 2, 32, 64, 64, 64, "bf16") == 0
    assert ws(1, 4096, 2, 32, 128, 128, 64, "bf16") == 0  # 1 is not a plan
    fake = 1 << 20
    st = kda.kda_chunk_fwd_with_plan(1, fake, fake, fake, fake, fake, None, None, 1, 64, 1, 1,
                                     32, 32, 16, "f32", fake, None, fake, 1 << 30, stream=0,
                                     check=False)
    assert st == kda.KDA_ERR_INVALID_ARG
    st = kda.kda_chunk_fwd_with_plan("split", fake, fake, fake, fake, fake, None, None, 1, 64, 1,
                                     1, 32, 32, 16, "f32", fake, None, fake, 1 << 30, stream=0,
                                     check=False)
    assert st == kda.KDA_ERR_UNSUPPORTED


def test_default_plan_ignores_the_environment(lib, monkeypatch):
    """The plan and the workspace size are functions of the arguments only."""
    f = kda.kda_chunk_fwd_workspace_size
    before = (f(4096, 2, 32, 128, 128, 64, "bf16"), kda.kda_chunk_fwd_plan(
        4096, 2, 32, 128, 128, 64, "bf16"))
    monkeypatch.setenv("KDA_CHUNK_PATH", "simt")
    after = (f(4096, 2, 32, 128, 128, 64, "bf16"), kda.kda_chunk_fwd_plan(
        4096, 2, 32, 128, 128, 64, "bf16"))
    assert before == after


def test_python_wrappers_reject_tensors_the_abi_would_misread(lib):
    """Checked in Python before any pointer reaches the library: a transposed
    (non-contiguous) view, a bf16 gate, q and v of different dtypes."""
    import torch
    T, H, d = 8, 2, 32
    q = torch.zeros(T, H, d, dtype=torch.bfloat16)
    g = torch.zeros(T, H, d)
    beta = torch.zeros(T, H)
    o = torch.zeros(T, H, d, dtype=torch.bfloat16)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    args = dict(initial_state=None, cu_seqlens=None, B=1, T=T, num_seqs=1, H=H, dk=d, dv=d,
                chunk=16, dtype="bf16", o=o, final_state=None, workspace=ws)
    with pytest.raises(ValueError, match="contiguous"):
        kda.kda_chunk_fwd(q.transpose(0, 1), q, q, g, beta, **args)
    with pytest.raises(ValueError, match="float32"):
        kda.kda_chunk_fwd(q, q, q, g.to(torch.bfloat16), beta, **args)
    with pytest.raises(ValueError, match="bfloat16"):
        kda.kda_chunk_fwd(q, q, q.float(), g, beta, **args)
    with pytest.raises(ValueError, match="float32"):
        kda.kda_decode_step(q[0], q[0], q[0], g[0], beta[0].to(torch.bfloat16),
                            torch.zeros(1, H, d, d), o[0], 1, H, d, d, "bf16")
    with pytest.raises(ValueError, match="contiguous"):
        kda.kda_decode_step(q[0], q[0], q[0], g[0], beta[0],
                            torch.zeros(1, H, d, d).transpose(2, 3), o[0], 1, H, d, d, "bf16")


def test_layer_decode_rejects_bad_arguments(lib):
    f, F = kda.kda_layer_decode_step, 1 << 20
    ptrs = [F] * 14
    ok = dict(N=2, H=2, dk=128, dv=128, dtype="bf16", l2_eps=1e-6, rms_eps=1e-6, y=F, stream=0,
              check=False)
    assert f(*ptrs, **dict(ok, dk=48)) == kda.KDA_ERR_UNSUPPORTED
    assert f(*ptrs, **dict(ok, rms_eps=0.0)) == kda.KDA_ERR_INVALID_ARG
    assert f(*ptrs, **dict(ok, N=-1)) == kda.KDA_ERR_INVALID_ARG
    assert f(*ptrs[:13], None, **ok) == kda.KDA_ERR_INVALID_ARG      # no w_norm
    assert f(*ptrs[:13], F + 4, **ok) == kda.KDA_ERR_INVALID_ARG     # misaligned
    assert f(*ptrs, **dict(ok, N=0)) == kda.KDA_OK


def test_layer_prefill_rejects_bad_arguments(lib):
    f, F = kda.kda_layer_chunk_fwd, 1 << 20
    ptrs = [F] * 10
    ok = dict(B=1, T=64, num_seqs=1, H=2, dk=128, dv=128, chunk=64, dtype="bf16", gate=F,
              w_norm=F, l2_eps=1e-6, rms_eps=1e-6, y=F, final_state=None, workspace=F,
              workspace_bytes=1 << 30, stream=0, check=False)
    assert f(*ptrs, **dict(ok, dk=48)) == kda.KDA_ERR_UNSUPPORTED
    assert f(*ptrs, **dict(ok, l2_eps=0.0)) == kda.KDA_ERR_INVALID_ARG
    assert f(*ptrs, **dict(ok, w_norm=None)) == kda.KDA_ERR_INVALID_ARG
    assert f(*ptrs, **dict(ok, y=F + 8)) == kda.KDA_ERR_INVALID_ARG
    assert f(*ptrs, **dict(ok, workspace=None)) == kda.KDA_ERR_WORKSPACE
    assert f(*ptrs, **dict(ok, workspace_bytes=16)) == kda.KDA_ERR_WORKSPACE
    assert kda.kda_layer_chunk_fwd_workspace_size(64, 1, 2, 128, 128, 64, "bf16") > 0
    assert kda.kda_layer_chunk_fwd_workspace_size(64, 1, 2, 48, 128, 64, "bf16") == 0


def test_binding_argument_counts_match_the_header(lib):
    """Every ctypes signature in the binding has as many arguments as the
    header's declaration of that function."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    from gated_delta_rule_124_b200 import kda as kmod
    for name, (args, _res) in kmod._SIGS.items():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", src)
        assert m, name
        params = [x for x in m.group(1).split(",") if x.strip() and x.strip() != "void"]
        assert len(params) == len(args), (name, len(params), len(args))
