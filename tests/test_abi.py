"""The C-ABI library builds, loads and exports every symbol its header declares;
host-side validation answers without touching a GPU.

The validation tests pass fabricated addresses that the library must reject
before any launch; they only run in a process that sees no CUDA device, so a
validation bug can never launch a kernel on them.  On a GPU machine the GPU
test at the end reruns them in a child process with no visible device; the GPU
parity tests repeat the rejections with real buffers.
"""
import ctypes
import os
import re
import subprocess
import sys

import pytest
import torch

import linear_attention_recurrent_decode_b200 as kda
from linear_attention_recurrent_decode_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda_decode.h")
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]
no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fabricated pointers: CPU-only check")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kda.library()


def declared_functions():
    """Every function the headers under include/ declare."""
    names = set()
    for path in HEADERS:
        text = open(path).read()
        names |= {re.findall(r"\w+", m)[-1] for m in re.findall(r"^KDA_API([^(;]*)\(", text, re.M)}
    return names


def test_header_declares_the_documented_entry_points():
    assert declared_functions() == {"kda_decode", "kda_decode_gated_rmsnorm", "kda_decode_bf16_state",
                                    "kda_decode_gated_rmsnorm_bf16_state", "kda_decode_ex",
                                    "kda_decode_host", "kda_decode_host_pipelined", "kda_status_string",
                                    "kda_abi_version", "kda_host_memory_is_mapped", "kda_decode_device_error",
                                    "kda_prefill", "kda_prefill_workspace_bytes", "kda_prefill_no_alloc",
                                    "kda_prefill_stage"}


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(kda.EXPORTED_SYMBOLS) == declared_functions()


def test_library_exports_nothing_else(lib):
    out = os.popen(f"nm -D --defined-only {kda.LIBRARY_PATH}").read()
    syms = {line.split()[-1] for line in out.splitlines() if line.split()[1] in ("T", "t")}
    assert {s for s in syms if s.startswith("kda_")} == declared_functions()


def test_status_strings_and_version(lib):
    assert kda.status_string(kda.KDA_OK) == "ok"
    for s in range(1, 8):
        assert kda.status_string(s) and kda.status_string(s) != "unknown status"
    assert kda.status_string(99) == "unknown status"
    assert lib.kda_abi_version() == (1 << 16) | 9


def test_device_error_query_validates_its_argument(lib):
    assert lib.kda_decode_device_error(None, 0) == kda.KDA_ERR_INVALID_ARG


# ----------------------------------------------------------------- validation
BASE = 1 << 40  # never dereferenced: every call below is rejected on the host


def call(lib, N=2, T=1, HV=2, K=128, V=128, q=None, k=None, v=None, g=None, beta=None,
         state=None, slot=None, out=None, gate=None, w=None, eps=1e-6, gated=False):
    step = 1 << 30
    ptr = dict(q=BASE, k=BASE + step, v=BASE + 2 * step, g=BASE + 3 * step, beta=BASE + 4 * step,
               state=BASE + 5 * step, slot=BASE + 8 * step, out=BASE + 9 * step,
               gate=BASE + 10 * step, w=BASE + 11 * step)
    for key, val in dict(q=q, k=k, v=v, g=g, beta=beta, state=state, slot=slot, out=out, gate=gate,
                         w=w).items():
        if val is not None:
            ptr[key] = val
    if gated:
        return lib.kda_decode_gated_rmsnorm(ptr["q"], ptr["k"], ptr["v"], ptr["g"], ptr["beta"],
                                            ptr["state"], ptr["slot"], ptr["gate"], ptr["w"], eps,
                                            ptr["out"], N, T, HV, K, V, 0.1, None)
    return lib.kda_decode(ptr["q"], ptr["k"], ptr["v"], ptr["g"], ptr["beta"], ptr["state"],
                          ptr["slot"], ptr["out"], N, T, HV, K, V, 0.1, None)


@no_gpu
@pytest.mark.parametrize("gated", [False, True])
def test_empty_batches_are_noops_without_pointers(lib, gated):
    assert call(lib, N=0, q=0, k=0, v=0, g=0, beta=0, state=0, slot=0, out=0, gate=0, w=0,
                gated=gated) == kda.KDA_OK
    assert call(lib, T=0, q=0, k=0, v=0, g=0, beta=0, state=0, slot=0, out=0, gate=0, w=0,
                gated=gated) == kda.KDA_OK


@no_gpu
@pytest.mark.parametrize("gated", [False, True])
def test_rejections(lib, gated):
    E = kda
    assert call(lib, N=-1, gated=gated) == E.KDA_ERR_INVALID_ARG
    assert call(lib, T=-2, gated=gated) == E.KDA_ERR_INVALID_ARG
    assert call(lib, HV=0, gated=gated) == E.KDA_ERR_UNSUPPORTED
    assert call(lib, K=0, gated=gated) == E.KDA_ERR_UNSUPPORTED
    assert call(lib, K=257, gated=gated) == E.KDA_ERR_UNSUPPORTED
    assert call(lib, K=512, gated=gated) == E.KDA_ERR_UNSUPPORTED
    assert call(lib, V=0, gated=gated) == E.KDA_ERR_UNSUPPORTED
    assert call(lib, q=0, gated=gated) == E.KDA_ERR_INVALID_ARG
    assert call(lib, slot=0, gated=gated) == E.KDA_ERR_INVALID_ARG
    assert call(lib, q=BASE + 8, gated=gated) == E.KDA_ERR_MISALIGNED
    assert call(lib, state=BASE + 5 * (1 << 30) + 4, gated=gated) == E.KDA_ERR_MISALIGNED
    assert call(lib, beta=BASE + 4 * (1 << 30) + 2, gated=gated) == E.KDA_ERR_MISALIGNED
    # out overlapping an input, or the pool
    assert call(lib, out=BASE + 64, gated=gated) == E.KDA_ERR_ALIAS
    assert call(lib, out=BASE + 5 * (1 << 30), gated=gated) == E.KDA_ERR_ALIAS
    # an input starting inside the pool's slot 0
    assert call(lib, g=BASE + 5 * (1 << 30) + 4096, gated=gated) == E.KDA_ERR_ALIAS
    if gated:
        assert call(lib, V=288, gated=True) == E.KDA_ERR_UNSUPPORTED  # 9 tiles > one cluster
        assert call(lib, gate=0, gated=True) == E.KDA_ERR_INVALID_ARG
        assert call(lib, w=BASE + 11 * (1 << 30) + 2, gated=True) == E.KDA_ERR_MISALIGNED
        assert call(lib, eps=-1.0, gated=True) == E.KDA_ERR_INVALID_ARG
        assert call(lib, eps=float("nan"), gated=True) == E.KDA_ERR_INVALID_ARG
        assert call(lib, eps=float("inf"), gated=True) == E.KDA_ERR_INVALID_ARG
        assert call(lib, out=BASE + 10 * (1 << 30), gated=True) == E.KDA_ERR_ALIAS


@no_gpu
def test_host_memory_is_never_mapped_without_a_device(lib):
    assert lib.kda_host_memory_is_mapped(BASE, 4096) == 0
    assert lib.kda_host_memory_is_mapped(None, 16) == 0
    assert lib.kda_host_memory_is_mapped(BASE, 0) == 0


@no_gpu
def test_valid_call_without_a_device_reports_device_error(lib):
    assert call(lib) == kda.KDA_ERR_DEVICE
    assert call(lib, gated=True) == kda.KDA_ERR_DEVICE


@no_gpu
@pytest.mark.parametrize("gated", [False, True])
def test_general_shapes_pass_validation(lib, gated):
    """K outside {64, 128, 256} and V not a multiple of 32 take the general
    (masked, element-wise) form: valid, with element alignment only."""
    E = kda
    for K, V in [(96, 100), (192, 130), (1, 1), (256, 33), (48, 128), (128, 17)]:
        assert call(lib, K=K, V=V, gated=gated) == E.KDA_ERR_DEVICE, (K, V)
    # element alignment suffices for the general form, not for the vectorised one
    assert call(lib, K=96, V=100, q=BASE + 2, gated=gated) == E.KDA_ERR_DEVICE
    assert call(lib, K=96, V=100, q=BASE + 1, gated=gated) == E.KDA_ERR_MISALIGNED
    assert call(lib, K=96, V=100, g=BASE + 3 * (1 << 30) + 2, gated=gated) == E.KDA_ERR_MISALIGNED
    assert call(lib, K=128, V=128, q=BASE + 2, gated=gated) == E.KDA_ERR_MISALIGNED
    if gated:
        assert call(lib, K=96, V=257, gated=True) == E.KDA_ERR_UNSUPPORTED  # 9 tiles > one cluster


def test_binding_refuses_cpu_tensors():
    from linear_attention_recurrent_decode_b200 import workloads

    w = workloads.make(N=1, T=1, HV=1, K=64, V=32, num_slots=1)
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_decode(w.q, w.k, w.v, w.g, w.beta, w.state, w.slot_idx)


@no_gpu
def test_size_limits_are_rejected_on_the_host(lib):
    # grid = N * HV * V/32 CTAs must fit in 2^31 - 1
    assert call(lib, N=1 << 28, HV=2, V=128) == kda.KDA_ERR_UNSUPPORTED
    # element counts that overflow int64
    assert call(lib, N=1 << 40, T=1 << 20, HV=1 << 10) == kda.KDA_ERR_UNSUPPORTED


def test_args_struct_layout_matches_the_header(tmp_path):
    """The ctypes mirror of kda_decode_args has the C compiler's field offsets."""
    fields = [f for f, _ in kda.DecodeArgs._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "kda_decode.h"\nint main(void) {\n'
                   + "".join(f'  printf("%zu\\n", offsetof(kda_decode_args, {f}));\n' for f in fields)
                   + '  printf("%zu\\n", sizeof(kda_decode_args));\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    os.system(f"gcc -std=c11 -I{os.path.dirname(HEADER)} -o {exe} {src}")
    got = [int(x) for x in os.popen(str(exe)).read().split()]
    want = [getattr(kda.DecodeArgs, f).offset for f in fields] + [ctypes.sizeof(kda.DecodeArgs)]
    assert got == want


@no_gpu
def test_ex_entry_point_validation(lib):
    E = kda
    step = 1 << 30

    def args(**kw):
        a = kda.DecodeArgs()
        N, T, HV, K, V = 2, 1, 2, 128, 128
        a.q, a.q_row_stride = BASE, HV * K
        a.k, a.k_row_stride = BASE + step, HV * K
        a.v, a.v_row_stride = BASE + 2 * step, HV * V
        a.g, a.g_row_stride = BASE + 3 * step, HV * K
        a.beta, a.beta_row_stride = BASE + 4 * step, HV
        a.state_pool, a.slot_idx, a.out = BASE + 5 * step, BASE + 8 * step, BASE + 9 * step
        a.N, a.T, a.HV, a.K, a.V, a.scale = N, T, HV, K, V, 0.1
        for key, val in kw.items():
            setattr(a, key, val)
        return lib.kda_decode_ex(ctypes.byref(a), None)

    assert lib.kda_decode_ex(None, None) == E.KDA_ERR_INVALID_ARG
    assert args() == E.KDA_ERR_DEVICE                                  # valid, no device here
    assert args(q_row_stride=255) == E.KDA_ERR_INVALID_ARG             # shorter than a row
    assert args(q_row_stride=260) == E.KDA_ERR_MISALIGNED              # not a multiple of 8
    assert args(q_row_stride=512, T=1, N=2) == E.KDA_ERR_DEVICE        # a padded packed row
    assert args(state_dtype=2) == E.KDA_ERR_INVALID_ARG
    assert args(state_layout=kda.KDA_LAYOUT_VK) == E.KDA_ERR_DEVICE     # [V, K] blocks, valid
    assert args(state_layout=2) == E.KDA_ERR_INVALID_ARG
    assert args(raw_gate=BASE + 10 * step) == E.KDA_ERR_INVALID_ARG    # raw gate mixed with g
    assert args(gate=BASE + 10 * step) == E.KDA_ERR_INVALID_ARG        # gate without norm_weight
    raw = dict(g=0, beta=0, raw_gate=BASE + 3 * step, raw_beta=BASE + 4 * step + 2,
               A_log=BASE + 11 * step, dt_bias=BASE + 12 * step)
    assert args(**raw) == E.KDA_ERR_DEVICE                             # raw form, 2-byte raw_beta is fine
    assert args(**{**raw, "dt_bias": BASE + 12 * step + 4}) == E.KDA_ERR_MISALIGNED
    assert args(**{**raw, "A_log": 0}) == E.KDA_ERR_INVALID_ARG
    # checked slots: a declared pool size and an optional status word
    status = BASE + 13 * step
    assert args(num_slots=-1) == E.KDA_ERR_INVALID_ARG
    assert args(num_slots=4, status=status) == E.KDA_ERR_DEVICE          # valid
    assert args(num_slots=4, status=status + 2) == E.KDA_ERR_MISALIGNED
    assert args(num_slots=4, status=BASE + 9 * step + 8) == E.KDA_ERR_ALIAS   # inside out
    assert args(num_slots=4, status=BASE + 5 * step + 8) == E.KDA_ERR_ALIAS   # inside the pool
    assert args(num_slots=4, status=BASE + 2 * step) == E.KDA_ERR_ALIAS       # on an input
    # with the pool's size declared, every slot's block counts for aliasing
    block = 2 * 128 * 128 * 4
    assert args(g=BASE + 5 * step + 3 * block) == E.KDA_ERR_DEVICE            # slot 3: unseen unchecked
    assert args(g=BASE + 5 * step + 3 * block, num_slots=4) == E.KDA_ERR_ALIAS
    assert args(g=BASE + 5 * step + 4 * block, num_slots=4) == E.KDA_ERR_DEVICE  # just past the pool
    # the general form takes [K][V] blocks and activated g, beta only
    assert args(V=100, v_row_stride=2 * 100) == E.KDA_ERR_DEVICE
    assert args(V=100, v_row_stride=2 * 100 + 3) == E.KDA_ERR_DEVICE  # any row stride
    assert args(V=100, v_row_stride=200, state_layout=kda.KDA_LAYOUT_VK) == E.KDA_ERR_UNSUPPORTED
    assert args(K=96, q_row_stride=192, k_row_stride=192, g_row_stride=192, **raw) == E.KDA_ERR_UNSUPPORTED


@no_gpu
def test_host_entry_point_validation(lib):
    """kda_decode_host validates its host staging before anything is enqueued."""
    E = kda
    step = 1 << 30
    a = kda.DecodeArgs()
    N, T, HV, K, V = 2, 1, 2, 128, 128
    a.q, a.q_row_stride = BASE, HV * K
    a.k, a.k_row_stride = BASE + step, HV * K
    a.v, a.v_row_stride = BASE + 2 * step, HV * V
    a.g, a.g_row_stride = BASE + 3 * step, HV * K
    a.beta, a.beta_row_stride = BASE + 4 * step, HV
    a.state_pool, a.slot_idx, a.out = BASE + 5 * step, BASE + 8 * step, BASE + 9 * step
    a.N, a.T, a.HV, a.K, a.V, a.scale = N, T, HV, K, V, 0.1
    host_in, dev_in, host_out = BASE + 20 * step, BASE + 21 * step, BASE + 22 * step

    def call(hin=host_in, din=dev_in, nbytes=4096, hout=host_out):
        return lib.kda_decode_host(ctypes.byref(a), hin, din, nbytes, hout, None)

    assert lib.kda_decode_host(None, host_in, dev_in, 4096, host_out, None) == E.KDA_ERR_INVALID_ARG
    assert call() == E.KDA_ERR_DEVICE                      # valid, no device here
    assert call(nbytes=-1) == E.KDA_ERR_INVALID_ARG
    assert call(hin=None) == E.KDA_ERR_INVALID_ARG
    assert call(din=None) == E.KDA_ERR_INVALID_ARG
    assert call(hin=None, din=None, nbytes=0) == E.KDA_ERR_DEVICE  # nothing to copy in
    assert call(hout=None) == E.KDA_ERR_INVALID_ARG
    assert call(din=BASE + 5 * step - 64, nbytes=128) == E.KDA_ERR_ALIAS  # staging runs into the pool

    # the pipelined form: two distinct streams and both events are required
    s1, s2, ev1, ev2 = BASE + 30 * step, BASE + 31 * step, BASE + 32 * step, BASE + 33 * step

    def pcall(st=s1, cs=s2, r=ev1, f=ev2, nbytes=4096):
        return lib.kda_decode_host_pipelined(ctypes.byref(a), host_in, dev_in, nbytes, host_out, st, cs, r, f)

    assert pcall(st=None) == E.KDA_ERR_INVALID_ARG
    assert pcall(cs=None) == E.KDA_ERR_INVALID_ARG
    assert pcall(cs=s1) == E.KDA_ERR_INVALID_ARG
    assert pcall(r=None) == E.KDA_ERR_INVALID_ARG
    assert pcall(f=None) == E.KDA_ERR_INVALID_ARG
    assert pcall(nbytes=-1) == E.KDA_ERR_INVALID_ARG
    assert pcall() == E.KDA_ERR_DEVICE                     # valid, no device here


@no_gpu
def test_prefill_validation(lib):
    """kda_prefill's host checks, with fabricated addresses (rejected before any launch)."""
    E = kda
    step = 1 << 30
    N, T, HV = 2, 100, 2
    need = lib.kda_prefill_workspace_bytes(N, T, HV, 128, 128)
    assert need == 256 + N * HV * 2 * 246272  # a header, then two chunks per (n, h) of 61,568 fp32 each
    assert lib.kda_prefill_workspace_bytes(N, T, HV, 128, 64) == -1
    assert lib.kda_prefill_workspace_bytes(-1, T, HV, 128, 128) == -1
    assert lib.kda_prefill_workspace_bytes(N, 0, HV, 128, 128) == 0

    def call(q=BASE, ws=BASE + 12 * step, wsb=None, out=BASE + 9 * step, K=128, V=128, n=N, t=T, g=BASE + 3 * step,
             beta=BASE + 4 * step):
        return lib.kda_prefill(q, BASE + step, BASE + 2 * step, g, beta, BASE + 5 * step, BASE + 8 * step, out,
                               ws, need if wsb is None else wsb, n, t, HV, K, V, 0.1, None)

    assert call() == E.KDA_ERR_DEVICE                         # valid, no device here
    assert call(n=0, q=0, ws=0, out=0) == E.KDA_OK            # nothing to do
    assert call(K=64) == E.KDA_ERR_UNSUPPORTED
    assert call(V=256) == E.KDA_ERR_UNSUPPORTED
    assert call(t=-1) == E.KDA_ERR_INVALID_ARG
    assert call(q=0) == E.KDA_ERR_INVALID_ARG
    assert call(ws=0) == E.KDA_ERR_INVALID_ARG
    assert call(wsb=need - 1) == E.KDA_ERR_INVALID_ARG
    assert call(q=BASE + 8) == E.KDA_ERR_MISALIGNED
    assert call(ws=BASE + 12 * step + 4) == E.KDA_ERR_MISALIGNED
    assert call(beta=BASE + 4 * step + 2) == E.KDA_ERR_MISALIGNED
    assert call(out=BASE + 64) == E.KDA_ERR_ALIAS             # out over q
    assert call(ws=BASE + 9 * step + 64) == E.KDA_ERR_ALIAS   # workspace over out
    assert call(ws=BASE + 5 * step - 1024) == E.KDA_ERR_ALIAS # workspace runs into the pool
    assert call(g=BASE + 5 * step + 4096) == E.KDA_ERR_ALIAS  # an input inside slot 0

    def stage(s, **kw):
        return lib.kda_prefill_stage(s, BASE, BASE + step, BASE + 2 * step, BASE + 3 * step, BASE + 4 * step,
                                     BASE + 5 * step, BASE + 8 * step, BASE + 9 * step, BASE + 12 * step, need,
                                     kw.get("n", N), T, HV, kw.get("K", 128), 128, 0.1, None)

    for s in (0, 1, 2):                                      # one kernel each, validated like the whole call
        assert stage(s) == E.KDA_ERR_DEVICE
        assert stage(s, K=64) == E.KDA_ERR_UNSUPPORTED
    assert stage(3) == E.KDA_ERR_INVALID_ARG
    assert stage(-1) == E.KDA_ERR_INVALID_ARG


@no_gpu
def test_prefill_no_alloc_validation(lib):
    """kda_prefill_no_alloc: sizes beyond its fixed scratch are refused before
    any device work; other sizes are validated as kda_prefill validates them."""
    E = kda
    step = 1 << 30

    def call(N=1, T=1000, HV=8, K=128, V=128, q=BASE):
        return lib.kda_prefill_no_alloc(q, BASE + step, BASE + 2 * step, BASE + 3 * step, BASE + 4 * step,
                                        BASE + 5 * step, BASE + 8 * step, BASE + 9 * step, N, T, HV, K, V, 0.1,
                                        None)

    assert call() == E.KDA_ERR_DEVICE                      # 128 chunks fit: valid, no device here
    assert call(T=1088) == E.KDA_ERR_DEVICE                # 136 chunks: the most that fit
    assert call(T=1089) == E.KDA_ERR_SCRATCH_LIMIT         # 144 chunks
    assert call(N=2, T=8192) == E.KDA_ERR_SCRATCH_LIMIT
    assert call(K=64) == E.KDA_ERR_UNSUPPORTED
    assert call(T=-1) == E.KDA_ERR_INVALID_ARG
    assert call(N=0, q=0) == E.KDA_OK
    assert kda.status_string(E.KDA_ERR_SCRATCH_LIMIT).startswith("sizes need more scratch")


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a machine with a GPU")
def test_host_validation_suite_with_no_visible_device():
    """Rerun every fabricated-pointer validation test of this file in a child
    process that sees no CUDA device: a call that passes validation stops at
    KDA_ERR_DEVICE there, so none can launch, and the rejections are checked in
    full on the GPU machine too."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                        os.path.abspath(__file__)], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout and " skipped" not in r.stdout, r.stdout[-1000:]
