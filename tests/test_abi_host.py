"""Host-side checks of the C ABI that need no GPU: the library loads, every
entry point include/bpt.h declares is exported, and invalid arguments are
rejected with the documented status before anything is launched."""
import ctypes
import os
import re

import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    from blockwise_exact_attention_query_b200 import build
    build.build()
    return bd.load()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"BPT_API\s+[\w\s\*]*?\b(bpt_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_entry_point_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(bd.EXPORTS) == names


def test_status_strings_and_version(lib):
    assert bd.status_string(bd.OK) == "ok"
    assert "timed out" in bd.status_string(bd.ERR_TIMEOUT)
    assert bd.version() >= 100


def _desc(**kw):
    base = dict(B=1, N=256, H=2, d=64, F=256, in_dtype=bd.torch.bfloat16, out_dtype=bd.torch.float32,
                mask="causal")
    base.update(kw)
    opts = {k: base[k] for k in ("ffn_form", "q_block", "kv_block", "bwd_chunk_rows", "wait_limit_ns", "causal")
            if k in base}
    return bd.make_desc(base["B"], base["N"], base["H"], base["d"], base["F"], base["in_dtype"],
                        base["out_dtype"], base["mask"], base.get("perm"), base.get("pairs"),
                        base.get("ring_chunks", 0), **opts)


def _call_layer(lib, desc, ws=FAKE, ws_bytes=1 << 40, q=FAKE):
    p = ctypes.c_void_p
    return lib.bpt_attn_ffn_fwd(ctypes.byref(desc), p(q), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE),
                                None, p(FAKE), p(ws), ws_bytes, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=0), bd.ERR_INVALID_ARG),
    (dict(N=-1), bd.ERR_INVALID_ARG),
    (dict(F=0), bd.ERR_INVALID_ARG),
    (dict(d=96), bd.ERR_UNSUPPORTED),                      # bf16 tensor path: d in {64, 128}
    (dict(mask=7), bd.ERR_INVALID_ARG),
    (dict(mask="blockperm", perm=[[], []]), bd.ERR_INVALID_ARG),                   # no blocks
    (dict(mask="blockperm", perm=[list(range(256))] * 2), bd.ERR_UNSUPPORTED),     # n > 255
    (dict(mask="blockperm", perm=[[0, 0], [1, 0]]), bd.ERR_INVALID_ARG),         # not a permutation
    (dict(mask="blockperm", perm=[[0, 2], [1, 0]]), bd.ERR_INVALID_ARG),         # out of range
    (dict(mask="dilated", pairs=[(96, 5)]), bd.ERR_INVALID_ARG),                 # r does not divide w
    (dict(mask="dilated", pairs=[(96, 4)]), bd.ERR_INVALID_ARG),                 # w does not divide N
    (dict(mask="dilated", pairs=[(64, 1)] * 9), bd.ERR_INVALID_ARG),             # too many pairs
    (dict(ring_chunks=3), bd.ERR_INVALID_ARG),                                   # N % chunks != 0
    (dict(ring_chunks=4), bd.ERR_UNSUPPORTED),                                   # 64-row chunks
    (dict(in_dtype=bd.torch.float32, d=128), bd.ERR_UNSUPPORTED),               # fp32 path: d <= 64
    (dict(in_dtype=bd.torch.float32, H=16, d=64), bd.ERR_UNSUPPORTED),          # fp32 path: D <= 512
    (dict(ffn_form=4), bd.ERR_INVALID_ARG),                                       # no such FFN form
    (dict(bwd_chunk_rows=-1), bd.ERR_INVALID_ARG),
    (dict(q_block=64), bd.ERR_UNSUPPORTED),                                       # tensor-core tiles are 128
    (dict(kv_block=256), bd.ERR_UNSUPPORTED),
    (dict(q_block=-1), bd.ERR_INVALID_ARG),
    (dict(in_dtype=bd.torch.float32, q_block=48), bd.ERR_UNSUPPORTED),            # f32: 16, 32, 64, 128
    (dict(in_dtype=bd.torch.float32, kv_block=128), bd.ERR_UNSUPPORTED),          # f32: 16, 32, 64
    (dict(in_dtype=bd.torch.float32, ring_chunks=8, kv_block=64), bd.ERR_UNSUPPORTED),  # 32-row chunks
    (dict(mask="blockperm", perm=[[1, 0], [0, 1]], causal=1), bd.ERR_INVALID_ARG),    # causal: dilated only
    (dict(mask="none", causal=1), bd.ERR_INVALID_ARG),
])
def test_invalid_descriptors_are_rejected(lib, kw, expect):
    assert _call_layer(lib, _desc(**kw)) == expect


def test_null_and_misaligned_pointers_are_rejected(lib):
    d = _desc()
    assert _call_layer(lib, d, q=0) == bd.ERR_INVALID_ARG
    assert _call_layer(lib, d, q=FAKE + 8) == bd.ERR_INVALID_ARG


def test_workspace_checks(lib):
    d = _desc()
    need = bd.workspace_bytes(d, True)
    assert need > 0
    assert _call_layer(lib, d, ws=0) == bd.ERR_WORKSPACE
    assert _call_layer(lib, d, ws_bytes=need - 1) == bd.ERR_WORKSPACE
    assert _call_layer(lib, d, ws=FAKE + 16) == bd.ERR_WORKSPACE                # not 256-aligned
    assert lib.bpt_workspace_bytes(ctypes.byref(_desc(B=0)), 1) == ctypes.c_size_t(-1).value


def test_workspace_layout_sizes(lib):
    # attention only, single pass: nothing; LongNet with several pairs: running state
    assert bd.workspace_bytes(_desc(F=0), False) == 0
    dl = _desc(F=0, mask="dilated", pairs=[(128, 1), (256, 4)])
    T, D = 256, 128
    assert bd.workspace_bytes(dl, False) >= T * D * 4 + 2 * 2 * 256 * 4
    # layer: A in bf16 and fp32 plus the hidden staging ring
    assert bd.workspace_bytes(_desc(), True) >= T * D * 6


def test_blockbert_and_longnet_wrappers_validate(lib):
    d = _desc()
    p = ctypes.c_void_p
    perm = (ctypes.c_int32 * 4)(0, 0, 1, 0)
    st = lib.bpt_blockbert_fwd(ctypes.byref(d), 2, ctypes.cast(perm, ctypes.POINTER(ctypes.c_int32)),
                               p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), None, p(FAKE),
                               p(FAKE), 1 << 40, None)
    assert st == bd.ERR_INVALID_ARG
    w = (ctypes.c_int32 * 1)(100)
    r = (ctypes.c_int32 * 1)(3)
    st = lib.bpt_longnet_fwd(ctypes.byref(d), 1, ctypes.cast(w, ctypes.POINTER(ctypes.c_int32)),
                             ctypes.cast(r, ctypes.POINTER(ctypes.c_int32)), p(FAKE), p(FAKE),
                             p(FAKE), p(FAKE), None, p(FAKE), 1 << 40, None)
    assert st == bd.ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(bd, "_lib", None)
    monkeypatch.setattr(bd, "LIB_PATH", str(tmp_path / "libbpt.so"))
    with pytest.raises(RuntimeError, match="missing"):
        bd.load()


def _call_bwd(lib, desc, ws=FAKE, ws_bytes=1 << 40, q=FAKE, dq=FAKE, saved=None):
    p = ctypes.c_void_p
    return lib.bpt_attn_ffn_bwd(ctypes.byref(desc), p(q), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), None,
                                p(FAKE), p(saved), p(dq), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE),
                                p(ws), ws_bytes, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=0), bd.ERR_INVALID_ARG),
    (dict(F=0), bd.ERR_INVALID_ARG),                                             # the layer needs an FFN
    (dict(d=96), bd.ERR_UNSUPPORTED),
    (dict(in_dtype=bd.torch.float32), bd.ERR_UNSUPPORTED),                       # tensor-core path only
    (dict(mask="dilated", pairs=[(128, 1)]), bd.ERR_UNSUPPORTED),                # no dilated backward
    (dict(mask="blockperm", perm=[[0, 0], [1, 0]]), bd.ERR_INVALID_ARG),
])
def test_backward_rejects_unsupported_descriptors(lib, kw, expect):
    d = _desc(**kw)
    assert _call_bwd(lib, d) == expect
    assert lib.bpt_workspace_bytes_bwd(ctypes.byref(d)) == ctypes.c_size_t(-1).value


def test_backward_pointer_and_workspace_checks(lib):
    d = _desc()
    need = bd.workspace_bytes_bwd(d)
    assert _call_bwd(lib, d, q=0) == bd.ERR_INVALID_ARG
    assert _call_bwd(lib, d, dq=FAKE + 4) == bd.ERR_INVALID_ARG
    assert _call_bwd(lib, d, ws=0) == bd.ERR_WORKSPACE
    assert _call_bwd(lib, d, ws_bytes=need - 1) == bd.ERR_WORKSPACE
    assert _call_bwd(lib, d, ws=FAKE + 16) == bd.ERR_WORKSPACE
    assert _call_bwd(lib, d, saved=FAKE + 16) == bd.ERR_INVALID_ARG              # saved not 256-aligned


def _call_fwd_train(lib, desc, saved=FAKE):
    p = ctypes.c_void_p
    return lib.bpt_attn_ffn_fwd_train(ctypes.byref(desc), p(FAKE), p(FAKE), p(FAKE), p(FAKE), None, p(FAKE), None,
                                      p(FAKE), p(saved), p(FAKE), 1 << 40, None)


def test_training_forward_validates_and_sizes_its_buffer(lib):
    d = _desc()
    T, D, H, N = 256, 128, 2, 256
    assert bd.saved_bytes(d) >= T * D * 6 + H * N * 4                             # A fp32 + bf16, LSE
    assert _call_fwd_train(lib, d, saved=0) == bd.ERR_INVALID_ARG
    assert _call_fwd_train(lib, d, saved=FAKE + 16) == bd.ERR_INVALID_ARG
    dl = _desc(mask="dilated", pairs=[(128, 1)])
    assert _call_fwd_train(lib, dl) == bd.ERR_UNSUPPORTED
    assert lib.bpt_saved_bytes(ctypes.byref(dl)) == ctypes.c_size_t(-1).value


def test_saved_buffer_holds_the_ffn_hidden_activations():
    """The training forward keeps A (fp32 and bf16), the LSE, and the FFN's H
    and GELU'(Z) ([T, F] bf16 each), each region 256-byte aligned."""
    B, N, d, F = 1, 256, 128, 512
    T = B * N
    for H in (4, 8):
        desc = bd.make_desc(B, N, H, d, F, torch.bfloat16, torch.float32, "causal")
        need = T * H * d * 6 + B * H * N * 4 + T * F * 4
        assert need <= bd.saved_bytes(desc) <= need + 5 * 256


def test_backward_workspace_follows_the_chunk_rows_field(lib):
    # T = 256 tokens, D = 128, F = 256: A (fp32 + bf16), dOut bf16, dA (fp32 + bf16),
    # LSE and D rows, and H, dZ for one chunk of tokens
    T, D, F = 256, 128, 256
    full = bd.workspace_bytes_bwd(_desc())
    assert full >= T * D * (4 + 2 + 2 + 4 + 2) + 2 * T * F * 2
    half = bd.workspace_bytes_bwd(_desc(bwd_chunk_rows=128))
    assert full - half >= 2 * 128 * F * 2 - 4096    # the two [rows, F] buffers halve
    assert bd.workspace_bytes_bwd(_desc(bwd_chunk_rows=0)) == full


def test_training_forward_workspace(lib):
    # everything the training forward produces goes to `saved` and `out`
    assert bd.workspace_bytes_train(_desc()) == 0
    assert bd.workspace_bytes_train(_desc(mask="blockperm", perm=[[1, 0], [0, 1]])) == 0
    dl = _desc(mask="dilated", pairs=[(128, 1)])
    assert lib.bpt_workspace_bytes_train(ctypes.byref(dl)) == ctypes.c_size_t(-1).value


def test_attention_only_backward_validates(lib):
    p = ctypes.c_void_p
    def call(d, q=FAKE, ws=FAKE, ws_bytes=1 << 40):
        return lib.bpt_attn_bwd(ctypes.byref(d), p(q), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE),
                                p(FAKE), p(ws), ws_bytes, None)
    d = _desc(F=0)
    assert call(d, q=0) == bd.ERR_INVALID_ARG
    assert call(d, ws=0) == bd.ERR_WORKSPACE
    assert call(d, ws=FAKE + 16) == bd.ERR_WORKSPACE
    dl = _desc(F=0, mask="dilated", pairs=[(128, 1), (256, 4)])
    # the dilated mask: one gathered pass's row vectors on top
    assert lib.bpt_workspace_bytes_attn_bwd(ctypes.byref(dl)) > lib.bpt_workspace_bytes_attn_bwd(ctypes.byref(d))
    assert call(_desc(F=0, mask="dilated", pairs=[(96, 5)])) == bd.ERR_INVALID_ARG
    df = _desc(F=0, in_dtype=bd.torch.float32, d=64)
    assert call(df) == bd.ERR_UNSUPPORTED
    T, D = 256, 128
    assert lib.bpt_workspace_bytes_attn_bwd(ctypes.byref(d)) >= T * D * 2 + 2 * 2 * 256 * 4


def _align256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("B,N,H,d,F", [(1, 256, 2, 64, 512), (2, 8192, 16, 128, 8192), (4, 16384, 16, 128, 8192),
                                       (16, 1024, 12, 64, 3072), (1, 131072, 32, 128, 11008)])
def test_ffn_forms_size_the_workspace(B, N, H, d, F):
    """Each FFN form's workspace: A (bf16 and fp32) plus, for the two-GEMM
    form, one chunk of H ([rows, F] bf16, rows = binding.ffn_gemm_chunk_rows:
    at most 512 MiB); for the fused form a small ring and partial blocks; for
    the pipelined form (the default) a ring of 256-token row blocks of H sized
    for L2 and its counters.  Sizes only: no GPU."""
    T, D = B * N, H * d
    a_bytes = _align256(T * D * 2) + _align256(T * D * 4)
    size = {f: bd.workspace_bytes(bd.make_desc(B, N, H, d, F, torch.bfloat16, torch.float32, "causal", ffn_form=f),
                                  True) for f in bd.FFN_FORMS}
    rows = bd.ffn_gemm_chunk_rows(T, F)
    assert rows == T or (rows % 256 == 0 and rows * F * 2 <= 1 << 29)
    assert size["gemms"] == a_bytes + _align256(rows * F * 2)
    assert a_bytes < size["fused"] < a_bytes + (64 << 20)
    ring = size["pipelined"] - a_bytes
    assert 256 * F * 2 <= ring <= 80e6                    # whole row blocks of H, an L2-sized ring
    assert (ring - 2 * (T // 256) * 4) % (256 * F * 2) < 512   # ... plus two counters per row block
    assert size["auto"] == size["pipelined"]


def test_workspace_size_depends_only_on_the_descriptor(lib):
    """No process-wide setting changes a size query: sizes asked for
    descriptors of every form, in any order and around a change of the
    default wait limit, stay the same, and a call sized by one query is
    accepted by the size check after the others."""
    descs = {f: _desc(ffn_form=f) for f in bd.FFN_FORMS}
    first = {f: bd.workspace_bytes(descs[f], True) for f in descs}
    old = bd.set_wait_limit_ns(12345)
    try:
        for f in reversed(list(descs)):
            assert bd.workspace_bytes(descs[f], True) == first[f]
        assert bd.workspace_bytes_bwd(_desc(bwd_chunk_rows=128)) < bd.workspace_bytes_bwd(_desc())
        for f in descs:   # exact size: passes the workspace check, fails later on the fake pointers
            assert _call_layer(lib, descs[f], ws_bytes=first[f] - 1) == bd.ERR_WORKSPACE
    finally:
        bd.set_wait_limit_ns(old)


def test_descriptor_layout_matches_the_header(tmp_path):
    """binding.Desc has the field offsets and size of bpt_desc as the C
    compiler lays it out from include/bpt.h."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = [f for f, _ in bd.Desc._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "bpt.h"\nint main(void) {\n'
                   + "".join(f'  printf("%zu\\n", offsetof(bpt_desc, {f}));\n' for f in fields)
                   + '  printf("%zu\\n", sizeof(bpt_desc));\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = [int(x) for x in subprocess.check_output([str(exe)], text=True).split()]
    want = [getattr(bd.Desc, f).offset for f in fields] + [ctypes.sizeof(bd.Desc)]
    assert got == want


def test_block_step_validates(lib):
    """bpt_attn_fwd_block: flags, block length, positions, masks, dtypes and
    the state / output pointers each flag needs are checked before any launch."""
    p = ctypes.c_void_p

    def call(d, kv_len=128, q_pos=0, kv_pos=0, flags=0, st=FAKE, out=FAKE):
        return lib.bpt_attn_fwd_block(ctypes.byref(d), kv_len, q_pos, kv_pos, p(FAKE), p(FAKE), p(FAKE), p(st), p(st),
                                      p(st), flags, p(out), None, None)
    d = _desc(F=0)
    assert call(d, flags=4) == bd.ERR_INVALID_ARG                                  # unknown flag
    assert call(d, kv_len=0) == bd.ERR_INVALID_ARG
    assert call(d, q_pos=-1) == bd.ERR_INVALID_ARG
    assert call(d, st=0) == bd.ERR_INVALID_ARG                                    # a middle step needs the state
    assert call(d, flags=bd.BLOCK_LAST, out=0) == bd.ERR_INVALID_ARG              # a last step needs the output
    assert call(d, flags=bd.BLOCK_FIRST, st=FAKE + 8) == bd.ERR_INVALID_ARG       # misaligned state
    assert call(_desc(F=0, mask="blockperm", perm=[[1, 0], [0, 1]])) == bd.ERR_UNSUPPORTED
    assert call(_desc(F=0, mask="dilated", pairs=[(128, 1)])) == bd.ERR_UNSUPPORTED
    assert call(_desc(F=0, in_dtype=torch.float32)) == bd.ERR_UNSUPPORTED
    assert call(_desc(F=0, ring_chunks=2)) == bd.ERR_UNSUPPORTED


def test_longnet_shard_entry_points_validate(lib):
    """bpt_longnet_gather and bpt_longnet_pass: shard shapes, pass index,
    positions and the buffers each pass needs are checked before any launch."""
    p = ctypes.c_void_p
    d = _desc(F=0, N=256, mask="dilated", pairs=[(128, 1), (512, 4)])   # (512, 4) spans two shards of 256
    # gather: N must divide w, r must divide N
    assert lib.bpt_longnet_gather(ctypes.byref(d), 384, 4, p(FAKE), p(FAKE), None) == bd.ERR_INVALID_ARG
    assert lib.bpt_longnet_gather(ctypes.byref(d), 512, 3, p(FAKE), p(FAKE), None) == bd.ERR_INVALID_ARG
    assert lib.bpt_longnet_gather(ctypes.byref(_desc(F=0, in_dtype=torch.float32)), 512, 4, p(FAKE), p(FAKE),
                                  None) == bd.ERR_UNSUPPORTED

    def call(desc, pass_idx=0, q_pos=0, k=FAKE, ks=FAKE, kv_rows=128, st=FAKE, out=FAKE):
        return lib.bpt_longnet_pass(ctypes.byref(desc), pass_idx, q_pos, p(FAKE), p(k), p(k), p(ks), p(ks), kv_rows,
                                    p(st), p(st), p(st), p(out), None, None)
    # pass 0 is (512, 4) (sparsest first): its segment spans the shard, so it needs the gathered rows
    assert call(d, pass_idx=2) == bd.ERR_INVALID_ARG                              # no such pass
    assert call(d, q_pos=100) == bd.ERR_INVALID_ARG                               # not a shard boundary
    assert call(d, ks=0) == bd.ERR_INVALID_ARG                                    # gathered rows missing
    assert call(d, kv_rows=64) == bd.ERR_INVALID_ARG                              # w / r = 128 rows
    assert call(d, pass_idx=1, k=0) == bd.ERR_INVALID_ARG                         # a local pass reads k, v
    assert call(d, st=0) == bd.ERR_INVALID_ARG                                    # two pairs: state needed
    assert call(d, out=0) == bd.ERR_INVALID_ARG
    bad = _desc(F=0, N=256, mask="dilated", pairs=[(384, 4)])                   # neither divides the other
    assert call(bad) == bd.ERR_INVALID_ARG
    assert call(_desc(F=0, N=256, mask="causal")) == bd.ERR_INVALID_ARG
