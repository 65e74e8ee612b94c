"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os

import pytest

import block_sparse_gqa_05_b200 as M
from block_sparse_gqa_05_b200 import msa as B


@pytest.fixture(scope="module")
def L():
    return B.lib()


def tiny(**kw):
    d = dict(batch=1, seq_q=2048, seq_kv=2048, q_offset=0, n_q_heads=8, n_kv_heads=2,
             head_dim=64, index_dim=32, block=128, topk=4)
    d.update(kw)
    return M.Shape(**d)


def test_exports_every_header_symbol(L):
    names = B.header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(8):
        s = L.msa_status_string(code).decode()
        assert s.startswith(B.STATUS[code])


def ws(shape, op):
    n = ctypes.c_size_t(123)
    st = B.lib().msa_workspace_size(ctypes.byref(shape), op, ctypes.byref(n))
    return st, n.value


def test_workspace_sizes_and_validation():
    st, n = ws(tiny(), M.OP_INDEX_SCORES)
    assert st == 0 and n == 0
    st, pre = ws(tiny(), M.OP_SPARSE_PREFILL)
    assert st == 0
    # partial outputs alone: B*T*H*k*d bf16 + B*T*H*k lse
    assert pre >= 2048 * 8 * 4 * 64 * 2 + 2048 * 8 * 4 * 4
    st, fwd = ws(tiny(), M.OP_FORWARD)
    # the prefill forward fuses the top-k into the index scores: the selection
    # is in the workspace, the pooled scores are not
    assert st == 0 and pre + 2048 * 2 * 4 * 4 <= fwd < pre + 2048 * 2 * 16 * 4
    dec = tiny(batch=3, seq_q=1, seq_kv=5000, q_offset=4999)
    st, n = ws(dec, M.OP_SPARSE_DECODE)
    assert st == 0 and n >= 3 * 8 * 4 * 64 * 4
    st, nd = ws(dec, M.OP_DENSE_DECODE)
    assert st == 0 and nd > 0
    # the alignment forward runs the prefill path for every T, decode shapes too
    st, al = ws(tiny(), M.OP_FORWARD_ALIGNMENT)
    assert st == 0 and al == fwd + 2048 * 2 * 16 * 4   # + the pooled scores the KL reads
    st, ald = ws(dec, M.OP_FORWARD_ALIGNMENT)
    st2, fd = ws(dec, M.OP_FORWARD)
    st3, pd = ws(dec, M.OP_SPARSE_PREFILL)
    assert st == st2 == st3 == 0 and ald >= pd and ald != fd
    # decode needs T == 1 and q_offset == N - 1
    assert ws(tiny(batch=3, seq_q=1, seq_kv=5000, q_offset=10), M.OP_SPARSE_DECODE)[0] == 1
    assert ws(tiny(), M.OP_SPARSE_DECODE)[0] == 1


def test_prefill_shared_memory_limits():
    # the combine keeps k x H (max, sum) pairs of a token on chip, the
    # inversion a 2 x nb histogram: shapes past one CTA's shared memory are
    # refused up front (decode, which uses neither, is not limited)
    many = dict(seq_q=256, seq_kv=4096, q_offset=3840, n_q_heads=1024, n_kv_heads=64, topk=64)
    for op in (M.OP_SPARSE_PREFILL, M.OP_FORWARD, M.OP_FORWARD_ALIGNMENT):
        assert ws(tiny(**many), op)[0] == 5
    assert ws(tiny(**dict(many, n_q_heads=256, n_kv_heads=16)), M.OP_FORWARD)[0] == 0
    n = 26000 * 128
    assert ws(tiny(seq_q=256, seq_kv=n, q_offset=n - 256), M.OP_FORWARD)[0] == 5
    assert ws(tiny(seq_q=1, seq_kv=n, q_offset=n - 1), M.OP_FORWARD)[0] == 0


@pytest.mark.parametrize("bad,code", [
    (dict(block=64), 5), (dict(topk=0), 1), (dict(topk=65), 5), (dict(head_dim=96), 5),
    (dict(index_dim=48), 5), (dict(n_q_heads=7), 1), (dict(n_q_heads=6), 5), (dict(n_kv_heads=3, n_q_heads=6), 5),
    (dict(n_q_heads=64, n_kv_heads=2), 5), (dict(q_offset=1), 1), (dict(seq_q=0), 1),
    (dict(batch=0), 1),
])
def test_shape_validation(bad, code):
    assert ws(tiny(**bad), M.OP_FORWARD)[0] == code


def test_pointer_checks_precede_device_use(L):
    s = tiny()
    ok = ctypes.c_void_p(1 << 20)           # never dereferenced: validation fails first
    mis = ctypes.c_void_p((1 << 20) + 8)
    assert L.msa_index_scores(ctypes.byref(s), None, ok, ok, None) == 2
    assert L.msa_index_scores(ctypes.byref(s), mis, ok, ok, None) == 3
    assert L.msa_block_topk(ctypes.byref(s), ok, None, None) == 2
    assert L.msa_sparse_attn_prefill(ctypes.byref(s), ok, ok, ok, ok, ok, None, None, 0, None) == 2
    assert L.msa_sparse_attn_prefill(ctypes.byref(s), ok, ok, ok, ok, ok, None, ok, 16, None) == 4
    bad = tiny(block=256)
    assert L.msa_forward(ctypes.byref(bad), ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40,
                         None) == 5
    # kl is required, 4-byte aligned, checked before the workspace
    assert L.msa_forward_alignment(ctypes.byref(s), ok, ok, ok, ok, ok, ok, None, None, None,
                                   ok, 1 << 40, None) == 2
    assert L.msa_forward_alignment(ctypes.byref(s), ok, ok, ok, ok, ok, ok, None, None,
                                   ctypes.c_void_p((1 << 20) + 2), ok, 1 << 40, None) == 3
    assert L.msa_forward_alignment(ctypes.byref(s), ok, ok, ok, ok, ok, ok, None, None, ok,
                                   ok, 16, None) == 4
    # paged decode: pool size, table pointer, then the ragged call's checks
    d1 = tiny(seq_q=1, seq_kv=4096, q_offset=0)
    paged = L.msa_forward_decode_paged
    assert paged(ctypes.byref(d1), 0, ok, ok, ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40,
                 None) == 1
    assert paged(ctypes.byref(d1), 1 << 30, ok, ok, ok, ok, ok, ok, ok, ok, None, None, ok,
                 1 << 40, None) == 5
    assert paged(ctypes.byref(d1), 8, ok, None, ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40,
                 None) == 2
    assert paged(ctypes.byref(d1), 8, ok, ctypes.c_void_p((1 << 20) + 2), ok, ok, ok, ok, ok, ok,
                 None, None, ok, 1 << 40, None) == 3
    assert paged(ctypes.byref(d1), 8, None, ok, ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40,
                 None) == 2
    assert paged(ctypes.byref(d1), 8, ok, ok, ok, ok, ok, ok, ok, ok, None, None, ok, 16,
                 None) == 4
    assert paged(ctypes.byref(tiny()), 8, ok, ok, ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40,
                 None) == 1                                # T must be 1
    # paged chunked prefill: pool size, table pointer and alignment, workspace
    pp = L.msa_forward_prefill_paged
    c1 = tiny(seq_q=256, seq_kv=4096, q_offset=3840)
    assert pp(ctypes.byref(c1), 0, ok, ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40, None) == 1
    assert pp(ctypes.byref(c1), 1 << 30, ok, ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40,
              None) == 5
    assert pp(ctypes.byref(c1), 8, None, ok, ok, ok, ok, ok, ok, None, None, ok, 1 << 40,
              None) == 2
    assert pp(ctypes.byref(c1), 8, ctypes.c_void_p((1 << 20) + 2), ok, ok, ok, ok, ok, ok, None,
              None, ok, 1 << 40, None) == 3
    assert pp(ctypes.byref(c1), 8, ok, ok, ok, ok, ok, ok, ok, None, None, ok, 16, None) == 4
    assert pp(ctypes.byref(tiny(seq_q=300, seq_kv=200)), 8, ok, ok, ok, ok, ok, ok, ok, None,
              None, ok, 1 << 40, None) == 1                # q_offset + T > N
    st, npp = ws(c1, M.OP_FORWARD_PREFILL_PAGED)
    st2, pre = ws(c1, M.OP_SPARSE_PREFILL)
    assert st == st2 == 0 and npp > pre                    # + the selection
    dec = tiny(seq_q=1, seq_kv=4096, q_offset=4095)
    assert L.msa_sparse_attn_decode(ctypes.byref(dec), ok, ok, ok, ok, ok, None, ok, 8, None) == 4
    assert L.msa_dense_attn_decode(ctypes.byref(s), ok, ok, ok, ok, None, ok, 1 << 30, None) == 1


def test_binding_rejects_cpu_tensors():
    import torch
    s = tiny()
    with pytest.raises(ValueError):
        M.index_scores(s, torch.zeros(1, 2048, 2, 32, dtype=torch.bfloat16),
                       torch.zeros(1, 2048, 32, dtype=torch.bfloat16),
                       pooled=torch.zeros(1, 2048, 2, 16))


def test_plain_c_caller(tmp_path):
    """tests/c_abi_host.c, compiled as C99 against include/msa.h and linked
    with libmsa, sizes workspaces and gets argument errors back as statuses."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "block_sparse_gqa_05_b200")
    exe = str(tmp_path / "c_abi_host")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(root, "include"), os.path.join(root, "tests", "c_abi_host.c"),
                    "-o", exe, os.path.join(pkg, "libmsa.so"), "-Wl,-rpath," + pkg],
                   check=True)
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
