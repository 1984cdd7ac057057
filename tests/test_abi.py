"""The C-ABI library loads, exports every symbol its header declares, and the
host-only entry points (workspace sizing, argument checks) behave as
documented.  No compute call is made here, so these run without a GPU."""

import ctypes
import os
import re

import pytest
import torch

from rnn_joint_network_02_b200 import frnnt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            names |= set(re.findall(r"FRNNT_API\s+[\w\s\*]*?\b(frnnt_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert {"frnnt_fwd_bwd", "frnnt_workspace_size", "frnnt_error_string", "frnnt_version"} <= declared
    lib = frnnt.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert set(frnnt.EXPORTED) <= declared


def test_version_and_error_strings():
    assert re.match(r"^\d+\.\d+\.\d+$", frnnt.version())
    for code in range(7):
        assert frnnt.error_string(code)
    assert "unknown" in frnnt.error_string(99)


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_workspace_size_is_host_only_and_positive(mode, dtype):
    d = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype=dtype, mode=mode)
    n = frnnt.workspace_size(d)
    assert n > 0


def test_tiled_workspace_bounded_by_chunk():
    big = frnnt.make_dims(8, 1500, 300, 512, 640, 640, 1024, mode="untiled")
    small = frnnt.make_dims(8, 1500, 300, 512, 640, 640, 1024, mode="tiled", chunk_cells=65536)
    assert frnnt.workspace_size(small) < frnnt.workspace_size(big) / 10


@pytest.mark.parametrize("field,value,code", [("B", 0, 2), ("H", -1, 2), ("blank", 8, 2), ("U", 1024, 2),
                                              ("U", 1023, 0), ("dtype", 7, 4), ("mode", 3, 4), ("path", 9, 4),
                                              ("wgrad_f32", 2, 2), ("wgrad_f32", 1, 0)])
def test_bad_dims_rejected(field, value, code):
    d = frnnt.make_dims(2, 12, 5, 16, 16, 32, 8, dtype="f32")
    setattr(d, field, value)
    n = ctypes.c_size_t(0)
    assert frnnt.lib().frnnt_workspace_size(ctypes.byref(d), ctypes.byref(n)) == code


def test_null_arguments_rejected_before_any_launch():
    lib = frnnt.lib()
    d = frnnt.make_dims(2, 12, 5, 16, 16, 32, 8, dtype="f32")
    nul = [None] * 17
    args = [ctypes.byref(d)] + nul[:6] + [None] * 3 + [None, None] + [None] * 6 + [None, 0, None, None]
    assert lib.frnnt_fwd_bwd(*args) == frnnt.FrnntError(1, "").code
    assert lib.frnnt_fwd_bwd(None, *args[1:]) == 1


def test_misaligned_pointer_rejected_before_any_launch():
    lib = frnnt.lib()
    d = frnnt.make_dims(2, 12, 5, 16, 16, 32, 8, dtype="f32")
    fake = [ctypes.c_void_p(4096 * (i + 1)) for i in range(20)]
    fake[0] = ctypes.c_void_p(4096 + 4)            # f misaligned
    args = ([ctypes.byref(d)] + fake[:6] + fake[6:9] + [None, fake[9]] + fake[10:16] +
            [fake[16], 1 << 40, fake[17], None])
    assert lib.frnnt_fwd_bwd(*args) == 6


def test_small_workspace_rejected_before_any_launch():
    lib = frnnt.lib()
    d = frnnt.make_dims(2, 12, 5, 16, 16, 32, 8, dtype="f32")
    fake = [ctypes.c_void_p(4096 * (i + 1)) for i in range(20)]
    args = ([ctypes.byref(d)] + fake[:6] + fake[6:9] + [None, fake[9]] + fake[10:16] +
            [fake[16], 16, fake[17], None])
    assert lib.frnnt_fwd_bwd(*args) == 3


def test_pruned_dims_rules():
    """prune_S: 0..32; pruned needs the bf16 tensor-core kernels; the plain
    entry refuses pruned dims and the pruned entry refuses unpruned ones."""
    lib = frnnt.lib()
    n = ctypes.c_size_t(0)
    d = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="bf16", prune_S=33)
    assert lib.frnnt_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 2
    d = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="f32", prune_S=4)
    assert lib.frnnt_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 4
    d = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="bf16", prune_S=4)
    assert lib.frnnt_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 0
    full = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="bf16", mode="untiled")
    pruned = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="bf16", mode="untiled", prune_S=4)
    assert frnnt.workspace_size(pruned) < frnnt.workspace_size(full)
    fake = [ctypes.c_void_p(4096 * (i + 1)) for i in range(20)]
    args = ([ctypes.byref(d)] + fake[:6] + fake[6:9] + [None, fake[9]] + fake[10:16] +
            [fake[16], 1 << 40, fake[17], None])
    assert lib.frnnt_fwd_bwd(*args) == 2            # pruned dims on the plain entry
    u = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="bf16")
    pargs = ([ctypes.byref(u)] + fake[:6] + fake[6:9] + [fake[19]] + [None, fake[9]] + fake[10:16] +
             [fake[16], 1 << 40, fake[17], None])
    assert lib.frnnt_fwd_bwd_pruned(*pargs) == 2    # unpruned dims on the pruned entry
    pargs[0] = ctypes.byref(d)
    pargs[10] = None                                # missing bounds
    assert lib.frnnt_fwd_bwd_pruned(*pargs) == 1


def test_tdt_dims_rules():
    """Duration sets: 2..8 strictly increasing frame counts starting 0, 1 and at
    most 8; the token-and-duration entry needs the bf16 tensor-core kernels, the
    marginal loss and the whole lattice; the plain entry refuses duration sets,
    the duration entry refuses dims without one, and a missing head is NULL."""
    lib = frnnt.lib()
    n = ctypes.c_size_t(0)

    def ws(**kw):
        args = dict(dtype="bf16", mode="untiled")
        args.update(kw)
        d = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, **args)
        return lib.frnnt_workspace_size(ctypes.byref(d), ctypes.byref(n))

    for bad in [(0,), (1, 2), (0, 2), (0, 1, 1), (0, 1, 3, 2), (0, 1, 9), tuple(range(8)) + (8,)][:6]:
        assert ws(durations=bad) == 2, bad
    assert ws(durations=(0, 1, 2, 3, 4)) == 0
    assert ws(durations=(0, 1, 2, 4, 8)) == 0
    assert ws(durations=tuple(range(8))) == 0
    assert ws(durations=(0, 1, 2), dtype="f32") == 4
    assert ws(durations=(0, 1, 2), loss="viterbi") == 4
    assert ws(durations=(0, 1, 2), prune_S=4) == 4
    with pytest.raises(ValueError):
        frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, durations=tuple(range(9)))
    plain = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="bf16")
    tdt = frnnt.make_dims(8, 100, 20, 256, 256, 256, 128, dtype="bf16", durations=(0, 1, 2))
    assert frnnt.workspace_size(tdt) > frnnt.workspace_size(plain)
    fake = [ctypes.c_void_p(4096 * (i + 1)) for i in range(24)]
    args = ([ctypes.byref(tdt)] + fake[:6] + fake[6:9] + [None, fake[9]] + fake[10:16] +
            [fake[16], 1 << 40, fake[17], None])
    assert lib.frnnt_fwd_bwd(*args) == 2                # duration set on the plain entry
    targs = ([ctypes.byref(plain)] + fake[:8] + fake[8:11] + [None, fake[11]] + fake[12:20] +
             [fake[20], 1 << 40, fake[21], None])
    assert lib.frnnt_fwd_bwd_tdt(*targs) == 2           # no duration set on the duration entry
    targs[0] = ctypes.byref(tdt)
    targs[7] = None                                     # missing W_d
    assert lib.frnnt_fwd_bwd_tdt(*targs) == 1


C_USER = r"""
#include <stdio.h>
#include <string.h>
#include "frnnt.h"
#include "frnnt_testing.h"

int main(void) {
  frnnt_dims d;
  size_t tiled = 0, untiled = 0;
  memset(&d, 0, sizeof d);
  d.B = 16; d.T = 400; d.U = 80; d.D_enc = 512; d.D_pred = 640; d.H = 640; d.V = 1024; d.blank = 0;
  d.dtype = FRNNT_BF16; d.mode = FRNNT_TILED; d.path = FRNNT_PATH_AUTO; d.loss = FRNNT_LOSS_MARGINAL;
  if (frnnt_workspace_size(&d, &tiled) != FRNNT_OK) return 2;
  d.mode = FRNNT_UNTILED;
  if (frnnt_workspace_size(&d, &untiled) != FRNNT_OK) return 3;
  d.blank = d.V;
  if (frnnt_workspace_size(&d, &untiled) != FRNNT_ERR_DIMS) return 4;
  if (frnnt_workspace_size(NULL, &untiled) != FRNNT_ERR_NULL) return 5;
  printf("%zu %zu %s|%s\n", tiled, untiled, frnnt_version(), frnnt_error_string(FRNNT_ERR_ALIGN));
  return 0;
}
"""


def test_headers_are_plain_c_and_host_calls_link(tmp_path):
    """The public headers compile as strict C11 (no C++ or CUDA types in the
    interface) and a C program linked against the library makes the host-only
    calls: workspace sizing for both modes, argument errors, strings."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    frnnt.lib()      # the library exists (raises with a build hint otherwise)
    src = tmp_path / "user.c"
    src.write_text(C_USER)
    exe = tmp_path / "user"
    libdir = os.path.dirname(frnnt.LIB_PATH)
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Wpedantic", "-Wstrict-prototypes", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lfrnnt",
                    "-Wl,-rpath," + libdir], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    tiled, untiled = int(out[0]), int(out[1])
    assert 0 < tiled < untiled, (tiled, untiled)
    size = ctypes.c_size_t(0)
    dims = frnnt.make_dims(16, 400, 80, 512, 640, 640, 1024, dtype="bf16", mode="untiled")
    assert frnnt.lib().frnnt_workspace_size(ctypes.byref(dims), ctypes.byref(size)) == frnnt.OK
    assert size.value == untiled, "C and Python callers see the same struct layout"
    assert out[2].startswith(frnnt.version()) and "aligned" in " ".join(out[2:])


def _tiny_args():
    from rnn_joint_network_02_b200 import synth
    b = synth.workload("tiny")
    return dict(f=b.f, g=b.g, W_f=b.W_f, W_g=b.W_g, W_o=b.W_o, b_o=b.b_o, labels=b.labels, T_len=b.T_len,
                U_len=b.U_len)


def _fwd_bwd(a, **kw):
    return frnnt.fwd_bwd(a["f"], a["g"], a["W_f"], a["W_g"], a["W_o"], a["b_o"], a["labels"], a["T_len"],
                         a["U_len"], **kw)


@pytest.mark.parametrize("field,bad,msg", [
    ("W_f", lambda t: t[:, :-1], "W_f has shape"),
    ("W_o", lambda t: t.t().contiguous(), "W_o|b_o|W_f"),
    ("labels", lambda t: t.long(), "labels is torch.int64"),
    ("labels", lambda t: t[:, :-1], "labels has shape"),
    ("T_len", lambda t: t[:1], "T_len has shape"),
    ("W_g", lambda t: t.double(), "W_g is torch.float64"),
    ("f", lambda t: t.transpose(0, 1).contiguous().transpose(0, 1), "f must be contiguous"),
])
def test_binding_rejects_bad_tensors_before_the_library(field, bad, msg):
    """Shapes, dtypes and layouts are checked on the host before any pointer
    reaches the library (a wrong one would be read out of bounds on the GPU)."""
    a = _tiny_args()
    a[field] = bad(a[field])
    with pytest.raises(ValueError, match=msg):
        _fwd_bwd(a)


def test_binding_rejects_host_tensors_and_bad_extras():
    a = _tiny_args()
    with pytest.raises(ValueError, match="CUDA tensors"):
        _fwd_bwd(a)
    with pytest.raises(ValueError, match="grad_loss is torch.float64"):
        _fwd_bwd(a, grad_loss=torch.ones(a["f"].shape[0], dtype=torch.float64))
    with pytest.raises(ValueError, match="bounds has shape"):
        frnnt.fwd_bwd_pruned(a["f"], a["g"], a["W_f"], a["W_g"], a["W_o"], a["b_o"], a["labels"], a["T_len"],
                             a["U_len"], torch.zeros(2, 3, dtype=torch.int32), 4)
    H = a["W_o"].shape[1]
    with pytest.raises(ValueError, match="b_d has shape"):
        frnnt.fwd_bwd_tdt(a["f"], a["g"], a["W_f"], a["W_g"], a["W_o"], a["b_o"], torch.zeros(5, H),
                          torch.zeros(4), a["labels"], a["T_len"], a["U_len"], (0, 1, 2, 3, 4))


def test_every_entry_point_is_documented_in_its_header():
    """Each FRNNT_API declaration directly follows a comment block (what the
    call computes, its arguments, ownership and errors)."""
    inc = os.path.join(ROOT, "include")
    seen = 0
    for fn in sorted(os.listdir(inc)):
        if not fn.endswith(".h"):
            continue
        lines = open(os.path.join(inc, fn)).read().splitlines()
        for i, line in enumerate(lines):
            m = re.search(r"FRNNT_API\s+[\w\s\*]*?\b(frnnt_\w+)\s*\(", line)
            if m:
                seen += 1
                assert i > 0 and lines[i - 1].strip().endswith("*/"), f"{fn}: {m.group(1)} has no doc comment"
    assert seen == len(_declared_functions())


def test_fp32_weight_gradient_outputs_are_one_flat_buffer():
    """With wgrad_f32 the binding lays dW_f, dW_g, dW_o, db_o out as fp32 views
    of one flat buffer, each segment on a 16-byte boundary (the library's
    alignment rule), so the data-parallel exchange reduces them in place."""
    import torch
    B, T, U, De, Dp, H, V = 2, 5, 3, 6, 5, 7, 9
    f = torch.zeros(B, T, De, dtype=torch.bfloat16)
    g = torch.zeros(B, U + 1, Dp, dtype=torch.bfloat16)
    W_f, W_g = torch.zeros(De, H, dtype=torch.bfloat16), torch.zeros(Dp, H, dtype=torch.bfloat16)
    W_o, b_o = torch.zeros(V, H, dtype=torch.bfloat16), torch.zeros(V, dtype=torch.bfloat16)
    dims = frnnt.make_dims(B, T, U, De, Dp, H, V, wgrad_f32=True)
    out = frnnt.Outputs(f, g, W_f, W_g, W_o, b_o, dims, with_workspace=False)
    assert out.df.dtype == torch.bfloat16 and out.dg.dtype == torch.bfloat16
    for name, ref in (("dW_f", W_f), ("dW_g", W_g), ("dW_o", W_o), ("db_o", b_o)):
        t = getattr(out, name)
        assert t.dtype == torch.float32 and tuple(t.shape) == tuple(ref.shape)
        assert t._base is out.wflat
        assert (t.data_ptr() - out.wflat.data_ptr()) % 16 == 0
