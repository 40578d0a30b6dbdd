"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

* libaq.so loads and exports every entry point include/aq.h declares;
* argument validation returns the documented status codes;
* view resolution folds uniform batch dims into rows and keeps the others as
  real batch dims with offsets from every stride (candle "Metal batched
  matmul" pitfall page; transformers issue #47331 shape table).
"""
import os
import re

import pytest
import torch

from group_wise_affine_qmv_b200 import aq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from group_wise_affine_qmv_b200 import build
    build.build()
    return aq.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "aq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(aq_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"aq_quantize", "aq_dequantize", "aq_qmv", "aq_qmm_t", "aq_qmm_t_grouped"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(aq.EXPORTED) <= set(names)


def test_status_strings(lib):
    assert lib.aq_status_string(0) == b"AQ_OK"
    assert lib.aq_status_string(6) == b"AQ_ERR_BITS"
    assert lib.aq_status_string(13) == b"AQ_ERR_TIMEOUT"
    assert lib.aq_version() >= 100


def _weights(N, K, bits, group, dtype=torch.bfloat16, batch=()):
    wq = torch.zeros(*batch, N, K * bits // 32, dtype=torch.int32)
    sc = torch.zeros(*batch, N, K // group, dtype=dtype)
    bi = torch.zeros(*batch, N, K // group, dtype=dtype)
    return wq, sc, bi


def plan(x, wq, sc, bi, group, bits, y=None, force_qmv=False):
    if y is None:
        y = torch.empty(tuple(x.shape[:-1]) + (wq.shape[-2],), dtype=x.dtype)
    return aq.aq_plan_linear(x, wq, sc, bi, group, bits, y, force_qmv)


def test_probe_shapes_fold_to_2d(lib):
    """[2,K], [2,1,K], [2,4,K], [1,S,K]: contiguous batch dims fold into rows."""
    K, N = 2048, 1024
    w = _weights(N, K, 4, 64)
    for shape, rows in [((2, K), 2), ((2, 1, K), 2), ((2, 4, K), 8), ((1, 7, K), 7), ((32, 1, K), 32), ((K,), 1)]:
        x = torch.zeros(shape, dtype=torch.bfloat16)
        p = plan(x, *w, 64, 4)
        assert p["nbatch_dims"] == 0 and p["M"] == rows and p["total_rows"] == rows, (shape, p)


def test_narrowed_q_heads_fold_but_batch_does_not(lib):
    """Q = qkv.narrow(1, 0, 4), strides [3840, 320, 64, 1]: heads fold (320 = 5*64),
    batch does not (3840 != 4*320) -> 2 launch batches x 20 rows, batch stride 3840."""
    qkv = torch.zeros(2, 12, 5, 64, dtype=torch.bfloat16)
    q = qkv.narrow(1, 0, 4)
    w = _weights(64, 64, 4, 64)
    y = torch.empty(2, 4, 5, 64, dtype=torch.bfloat16)
    p = plan(q, *w, 64, 4, y=y)
    assert p["M"] == 20 and p["nbatch_dims"] == 1
    assert p["batch_shape"] == (1, 2) and p["x_batch_stride"][1] == 3840 and p["x_row_stride"] == 64
    assert p["y_batch_stride"][1] == 4 * 5 * 64


def test_narrowed_linear4d(lib):
    """x = narrow(1, 0, 2) of [2,4,3,1408]: dims 1-2 fold (4224 = 3*1408), dim 0 does not."""
    base = torch.zeros(2, 4, 3, 1408, dtype=torch.bfloat16)
    x = base.narrow(1, 0, 2)
    w = _weights(2816, 1408, 8, 32)
    p = plan(x, *w, 32, 8)
    assert p["M"] == 6 and p["nbatch_dims"] == 1 and p["batch_shape"] == (1, 2)
    assert p["x_batch_stride"][1] == 16896 and p["x_row_stride"] == 1408


def test_batched_weights_keep_every_batch_dim(lib):
    """Scores case: per-(b,h) weight bank [2,4,5,...]: no dim may fold into rows."""
    qkv = torch.zeros(2, 12, 5, 64, dtype=torch.bfloat16)
    q = qkv.narrow(1, 0, 4)
    w = _weights(5, 64, 8, 64, batch=(2, 4))
    y = torch.empty(2, 4, 5, 5, dtype=torch.bfloat16)
    p = plan(q, *w, 64, 8, y=y)
    assert p["w_batched"] and p["M"] == 5 and p["nbatch_dims"] == 2
    assert p["batch_shape"] == (2, 4) and p["x_batch_stride"] == (3840, 320)
    assert p["w_batch_stride"] == (4 * 5 * 16, 5 * 16) and p["regime"] == "qmv"


def test_broadcast_weight_dim_folds(lib):
    """W [1, N, Kw] broadcast over x [3, 5, K]: the batch dim folds into rows."""
    x = torch.zeros(3, 5, 128, dtype=torch.bfloat16)
    w = _weights(16, 128, 4, 32, batch=(1,))
    p = plan(x, *w, 32, 4)
    assert p["M"] == 15 and p["nbatch_dims"] == 0 and not p["w_batched"]


def test_strided_rows_kept(lib):
    """A row-strided 2D x (every other row) keeps its row stride."""
    base = torch.zeros(8, 256, dtype=torch.bfloat16)
    x = base[::2]
    w = _weights(32, 256, 4, 64)
    p = plan(x, *w, 64, 4)
    assert p["M"] == 4 and p["x_row_stride"] == 512


def test_regime_by_rows(lib):
    w = _weights(1024, 1024, 4, 64)
    for x in (torch.zeros(1, 1024, dtype=torch.bfloat16), torch.zeros(4, 1, 1024, dtype=torch.bfloat16)):
        p = plan(x, *w, 64, 4)
        assert p["regime"] == "qmv" and p["kernel"] == "gemv"
    # forced GEMV whatever the size
    p = plan(torch.zeros(32, 1, 1024, dtype=torch.bfloat16), *w, 64, 4, force_qmv=True)
    assert p["regime"] == "qmv" and p["kernel"] == "gemv"


def test_plan_struct_layout(lib, tmp_path):
    """The ctypes mirrors of aq_plan and aq_view match the C declarations in include/aq.h field by
    field (sizes and offsets printed by a C program compiled against the header)."""
    import ctypes
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = [("aq_plan", aq.AqPlan), ("aq_view", aq.AqView)]
    body = ""
    for cname, cls in structs:
        body += f'  printf("%zu\\n", sizeof({cname}));\n'
        body += "".join(f'  printf("%zu\\n", offsetof({cname}, {f[0]}));\n' for f in cls._fields_)
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"aq.h\"\nint main(void) {\n" + body +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    expect = []
    for _, cls in structs:
        expect += [ctypes.sizeof(cls)] + [getattr(cls, f[0]).offset for f in cls._fields_]
    assert out == expect
    assert aq.AqPlan.kernel.offset == aq.AqPlan.nbatch_dims.offset + 4
    assert set(aq.KERNEL_NAMES.values()) == {"gemv", "warp_mma", "tc_small_m", "tc_prefill"}
    hdr = open(os.path.join(ROOT, "include", "aq.h")).read()
    for name, value in (("AQ_KERNEL_GEMV", 0), ("AQ_KERNEL_WARP_MMA", 1), ("AQ_KERNEL_TC_SMALL_M", 2),
                        ("AQ_KERNEL_TC_PREFILL", 3)):
        assert f"{name} = {value}" in hdr


@pytest.mark.parametrize("case,status", [
    ("bits", "AQ_ERR_BITS"), ("group", "AQ_ERR_GROUP"), ("kmod", "AQ_ERR_GROUP"), ("wshape", "AQ_ERR_SHAPE"),
    ("sshape", "AQ_ERR_SHAPE"), ("ydtype", "AQ_ERR_DTYPE"), ("sdtype", "AQ_ERR_DTYPE"), ("xdtype", "AQ_ERR_DTYPE"),
    ("stride", "AQ_ERR_STRIDE"), ("yshape", "AQ_ERR_SHAPE"), ("overlap", "AQ_ERR_OVERLAP"), ("rank", "AQ_ERR_RANK"),
    ("wbatch", "AQ_ERR_SHAPE"), ("align", "AQ_ERR_ALIGN"), ("yexpand", "AQ_ERR_OVERLAP"),
    ("yrows", "AQ_ERR_OVERLAP"), ("ybatch0", "AQ_ERR_OVERLAP"),
])
def test_validation_errors(lib, case, status):
    K, N, G, B = 256, 64, 64, 4
    x = torch.zeros(2, K, dtype=torch.bfloat16)
    wq, sc, bi = _weights(N, K, B, G)
    y = torch.empty(2, N, dtype=torch.bfloat16)
    bits, group = B, G
    if case == "bits":
        bits = 7
    elif case == "group":
        group = 16
    elif case == "kmod":
        x = torch.zeros(2, 96, dtype=torch.bfloat16)
        wq, sc, bi = _weights(N, 96, 4, 32)
        wq = torch.zeros(N, 12, dtype=torch.int32)
        group = 64
    elif case == "wshape":
        wq = torch.zeros(N, K * B // 32 + 1, dtype=torch.int32)
    elif case == "sshape":
        sc = torch.zeros(N, K // G + 1, dtype=torch.bfloat16)
    elif case == "ydtype":
        y = torch.empty(2, N, dtype=torch.float16)
    elif case == "sdtype":
        sc = sc.to(torch.float16)
    elif case == "xdtype":
        x = x.float()
    elif case == "stride":
        x = torch.zeros(K, 2, dtype=torch.bfloat16).t()
    elif case == "yshape":
        y = torch.empty(2, N + 1, dtype=torch.bfloat16)
    elif case == "overlap":
        buf = torch.zeros(2 * K, dtype=torch.bfloat16)
        x = buf.view(2, K)
        y = buf[: 2 * N].view(2, N)
    elif case == "rank":
        x = torch.zeros(1, 1, 1, 2, K, dtype=torch.bfloat16)
        with pytest.raises(ValueError):
            aq.view(x)
        return
    elif case == "wbatch":
        wq, sc, bi = _weights(N, K, B, G, batch=(3,))
    elif case == "align":
        wq = torch.zeros(N * (K * B // 32) + 1, dtype=torch.int32)[1:].view(N, K * B // 32)
    elif case == "yexpand":     # an expand()ed y: both rows are the same memory
        y = torch.empty(1, N, dtype=torch.bfloat16).expand(2, N)
    elif case == "yrows":       # row stride smaller than the row: rows overlap
        y = torch.empty(2 * N, dtype=torch.bfloat16).as_strided((2, N), (N // 2, 1))
    elif case == "ybatch0":     # a batch dim of stride 0 on a 3D y
        x = torch.zeros(3, 2, K, dtype=torch.bfloat16)
        y = torch.empty(1, 2, N, dtype=torch.bfloat16).expand(3, 2, N)
    with pytest.raises(aq.AQError) as ei:
        aq.aq_plan_linear(x, wq, sc, bi, group, bits, y)
    assert ei.value.name == status, (case, str(ei.value))


def test_empty_inputs_plan(lib):
    x = torch.zeros(0, 256, dtype=torch.bfloat16)
    w = _weights(64, 256, 4, 64)
    p = plan(x, *w, 64, 4)
    assert p["total_rows"] == 0


def test_output_self_overlap_rejected_everywhere(lib):
    """No output view may alias itself: quantize's outputs, dequantize's output and the grouped
    entry's y_sorted are checked like aq_qmm_t's y (before anything would launch)."""
    K, N, G, B = 256, 64, 64, 4
    w = torch.zeros(N, K, dtype=torch.float32)
    wq, sc, bi = _weights(N, K, B, G)
    lib_ = aq.load_library()
    bad_sc = torch.zeros(1, K // G, dtype=torch.bfloat16).expand(N, K // G)
    st = lib_.aq_quantize(aq.view(w), G, B, aq.view(wq), aq.view(bad_sc), aq.view(bi), None)
    assert lib_.aq_status_string(st) == b"AQ_ERR_OVERLAP"
    bad_w = torch.zeros(1, K, dtype=torch.float32).expand(N, K)
    st = lib_.aq_dequantize(aq.view(wq), aq.view(sc), aq.view(bi), G, B, aq.view(bad_w), None)
    assert lib_.aq_status_string(st) == b"AQ_ERR_OVERLAP"
    E, T = 2, 6
    xs = torch.zeros(T, K, dtype=torch.bfloat16)
    wqb, scb, bib = _weights(N, K, B, G, batch=(E,))
    ys = torch.zeros(1, N, dtype=torch.bfloat16).expand(T, N)
    st = lib_.aq_qmm_t_grouped(aq.view(xs), 8, E, aq.view(wqb), aq.view(scb), aq.view(bib), G, B, aq.view(ys),
                               None)
    assert lib_.aq_status_string(st) == b"AQ_ERR_OVERLAP"
    # a y whose zero stride sits on a dimension of extent 1 is fine
    y1 = torch.empty(1, N, dtype=torch.bfloat16).as_strided((1, N), (0, 1))
    assert aq.aq_plan_linear(torch.zeros(1, K, dtype=torch.bfloat16), wq, sc, bi, G, B, y1)["total_rows"] == 1
