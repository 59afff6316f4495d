"""C-ABI checks that need no GPU: the library loads, exports every function that include/svd.h
declares, sizes its workspace, names its status codes and rejects bad arguments before any
launch.  No compute call is made here."""
import ctypes
import math
import os
import re

import pytest

from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import build as svd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svd.h")
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def L():
    svd_build.build()
    return api.lib()


def declared_functions():
    src = "\n".join(open(h).read() for h in HEADERS)
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(svd_[a-z_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("svd_length_head", "svd_verify", "svd_distill_loss_grad", "svd_verify_distill",
              "svd_workspace_bytes", "svd_get_device_error", "svd_status_string"):
        assert n in names, n


def test_every_declared_symbol_is_exported(L):
    raw = ctypes.CDLL(api.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(raw, n)]
    assert not missing, missing


def test_workspace_bytes(L):
    a = L.svd_workspace_bytes(128, 16, 16, 256)
    b = L.svd_workspace_bytes(128, 16, 17, 256)
    c = L.svd_workspace_bytes(128, 16, 16, 0)
    assert a % 256 == 0 and a > 0
    assert b > a and c < a
    assert L.svd_workspace_bytes(-1, 16, 16, 0) == 0
    # header (256) + row records (32 B each) + per-sequence losses + head partials
    assert a >= 256 + 32 * 128 * 16 + 4 * 128 + 4 * 4 * 128


def test_status_strings(L):
    for code, name in api.STATUS_NAMES.items():
        assert L.svd_status_string(code).decode() == name
    assert L.svd_status_string(99).decode() == "SVD_ERR_UNKNOWN"


def test_argument_errors_return_before_launch(L):
    P = ctypes.c_void_p
    fake = P(0x1000)   # never dereferenced: validation fails first
    # k out of range
    assert L.svd_verify(fake, fake, None, fake, 4, 0, 0, 1024, 0, 1.0, 0, 0, fake, fake, fake,
                        None, fake, 1 << 20, None) == 1
    assert L.svd_verify(fake, fake, None, fake, 4, 33, 33, 1024, 0, 1.0, 0, 0, fake, fake, fake,
                        None, fake, 1 << 20, None) == 1
    # kt not in {k, k+1}
    assert L.svd_verify(fake, fake, None, fake, 4, 8, 10, 1024, 0, 1.0, 0, 0, fake, fake, fake,
                        None, fake, 1 << 20, None) == 1
    # V too large
    assert L.svd_verify(fake, fake, None, fake, 4, 8, 8, 10 ** 6, 0, 1.0, 0, 0, fake, fake, fake,
                        None, fake, 1 << 20, None) == 6
    # stochastic mode needs draft tokens
    assert L.svd_verify(fake, fake, None, fake, 4, 8, 8, 1024, 1, 1.0, 0, 0, fake, fake, fake,
                        None, P(0x10000), 1 << 20, None) == 1
    # bad temperature
    assert L.svd_verify(fake, fake, None, fake, 4, 8, 8, 1024, 0, 0.0, 0, 0, fake, fake, fake,
                        None, P(0x10000), 1 << 20, None) == 1
    # misaligned workspace, then too small a workspace
    assert L.svd_verify(fake, fake, None, fake, 4, 8, 8, 1024, 0, 1.0, 0, 0, fake, fake, fake,
                        None, P(0x10010), 1 << 20, None) == 2
    assert L.svd_verify(fake, fake, None, fake, 4, 8, 8, 1024, 0, 1.0, 0, 0, fake, fake, fake,
                        None, P(0x10000), 16, None) == 3
    # lambda outside [0,1], negative clip, NaN clip
    for lam, c in ((1.5, 1.0), (0.5, -1.0), (0.5, math.nan)):
        assert L.svd_distill_loss_grad(fake, fake, fake, 4, 8, 8, 1024, lam, c, 1.0, 1.0, None,
                                       fake, fake, 0, P(0x10000), 1 << 20, None) == 1
    # length head: bad gamma / rounding mode
    assert L.svd_length_head(fake, fake, None, fake, 0.0, 4, 256, 64, 8, 0.0, 0, None, fake,
                             P(0x10000), 1 << 20, None) == 1
    assert L.svd_length_head(fake, fake, None, fake, 0.0, 4, 256, 64, 8, 1.0, 7, None, fake,
                             P(0x10000), 1 << 20, None) == 1
    # empty batch: nothing to do, nothing launched
    assert L.svd_verify(None, None, None, None, 0, 8, 8, 1024, 0, 1.0, 0, 0, None, None, None,
                        None, None, 0, None) == 0
    assert L.svd_workspace_reset(None, 0, None) == 1
    assert L.svd_get_device_error(None, None) == 1
    assert L.svd_verify_distill(None, None, 0, None) == 1


def test_fused_args_struct_matches_header():
    # field count of svd_verify_distill_args in the header == ctypes mirror
    src = open(HEADER).read()
    body = src[src.index("typedef struct svd_verify_distill_args"):src.index("} svd_verify_distill_args;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    decls = [d.strip() for d in body.split("{", 1)[1].split(";") if d.strip()]
    n = sum(len(d.split(",")) for d in decls)
    assert n == len(api.VerifyDistillArgs._fields_)


def test_vocab_header_declares_the_sharded_calls():
    names = declared_functions()
    for n in ("svd_vs_stats", "svd_vs_resolve", "svd_vs_finish", "svd_vs_exchange_bytes",
              "svd_vs_workspace_bytes"):
        assert n in names, n


def _c_layout(struct, fields, tmp_path):
    """sizeof and field offsets of a header struct, from a C program built with gcc."""
    import subprocess
    src = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "svd_vocab.h"', "int main(void) {",
             '  printf("%%zu\\n", sizeof(%s));' % struct]
    for f in fields:
        lines.append('  printf("%%zu\\n", offsetof(%s, %s));' % (struct, f))
    lines.append("  return 0;\n}")
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    return int(out[0]), [int(x) for x in out[1:]]


@pytest.mark.parametrize("struct,mirror", [("svd_vs_args", api.VsArgs),
                                           ("svd_verify_distill_args", api.VerifyDistillArgs),
                                           ("svd_head_update_args", api.HeadUpdateArgs)])
def test_ctypes_mirrors_match_the_c_layout(struct, mirror, tmp_path):
    names = [f[0] for f in mirror._fields_]
    size, offs = _c_layout(struct, [("lambda" if n == "lambda_" else n) for n in names], tmp_path)
    assert size == ctypes.sizeof(mirror)
    assert offs == [getattr(mirror, n).offset for n in names]


def test_vocab_sizes_and_argument_errors(L):
    assert L.svd_vs_exchange_bytes(128, 17, 1) == 128 * 17 * 48
    assert L.svd_vs_exchange_bytes(128, 17, 2) == 128 * 17 * 32
    assert L.svd_vs_exchange_bytes(128, 17, 3) == 0
    assert L.svd_vs_workspace_bytes(4, 8, 10) == 0
    assert L.svd_vs_workspace_bytes(128, 16, 17) > 128 * 17 * 64
    fake = ctypes.c_void_p(0x1000)   # never dereferenced: validation fails first
    ws = ctypes.c_void_p(0x10000)

    def args(**kw):
        a = api.VsArgs()
        a.D = a.T = a.bk = a.accept_len = a.emitted = a.n_emitted = a.dlogits = a.loss_total = fake
        a.B, a.k, a.kt, a.V, a.v0, a.Vl, a.P, a.rank = 4, 8, 8, 1024, 0, 512, 2, 0
        a.mode, a.temperature, a.distill, a.lambda_, a.clip_c, a.grad_scale = 0, 1.0, 1, 0.5, 1.0, 1.0
        for k, v in kw.items():
            setattr(a, k, v)
        return ctypes.byref(a)

    bad = [dict(P=0), dict(rank=2), dict(rank=-1), dict(v0=600), dict(Vl=0), dict(k=33, kt=33),
           dict(kt=10), dict(mode=1), dict(temperature=0.0), dict(lambda_=2.0),
           dict(clip_c=-1.0), dict(distill=2), dict(D=None), dict(dlogits=None)]
    for kw in bad:
        assert L.svd_vs_stats(args(**kw), fake, ws, 1 << 20, None) == 1, kw
        assert L.svd_vs_resolve(args(**kw), fake, fake, ws, 1 << 20, None) == 1, kw
        assert L.svd_vs_finish(args(**kw), fake, ws, 1 << 20, None) == 1, kw
    # buffers and workspace
    assert L.svd_vs_stats(args(), None, ws, 1 << 20, None) == 1
    assert L.svd_vs_resolve(args(), fake, None, ws, 1 << 20, None) == 1
    assert L.svd_vs_finish(args(), None, ws, 1 << 20, None) == 1
    assert L.svd_vs_stats(args(), fake, ctypes.c_void_p(0x10010), 1 << 20, None) == 2
    assert L.svd_vs_stats(args(), fake, ws, 16, None) == 3
    # empty batch: nothing to do
    assert L.svd_vs_stats(args(B=0), None, None, 0, None) == 0
    assert L.svd_vs_stats(None, fake, ws, 1 << 20, None) == 1
