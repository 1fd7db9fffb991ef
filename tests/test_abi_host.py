"""Host-side checks of the C ABI: the library loads, exports every function its header
declares, and rejects bad arguments on the host before enqueueing anything.  No kernel
runs here.  The invalid calls use fake device addresses, so these tests are skipped when
a GPU is visible: if a check ever let one of them through, it must not reach a kernel."""
import ctypes

import pytest

import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import build

ERR_ARG, ERR_RANGE, ERR_WS, ERR_CUDA, ERR_UNSUP = -1, -2, -3, -4, -5
FAKE = 0x10000  # 16-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return pkv.lib()


def _no_gpu():
    import torch
    return not torch.cuda.is_available()


host_only = pytest.mark.skipif(not _no_gpu(), reason="fake-pointer calls run only without a GPU")


def test_exports_every_declared_symbol(lib):
    names = pkv.declared_functions()
    assert {"paged_kv_write", "paged_attention_decode", "copy_blocks",
            "paged_attention_decode_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/pagedkv.h but not exported"


def test_status_strings(lib):
    for code in (0, ERR_ARG, ERR_RANGE, ERR_WS, ERR_CUDA, ERR_UNSUP, 99):
        assert lib.pkv_status_string(code)


def test_partition_and_workspace_sizes(lib):
    # requested partition sizes are honoured; the automatic one is a multiple of 16, or 0
    # while the process runs the work-balanced split
    assert pkv.paged_attention_decode_partition_size(8, 8, 131073, 16, 512) == 512
    for B, Hkv, L in [(64, 40, 2049), (256, 8, 4097), (8, 8, 131073), (128, 8, 1281), (4, 4, 34),
                      (4096, 8, 2049)]:
        P = pkv.paged_attention_decode_partition_size(B, Hkv, L, 16, 0)
        assert P > 0 and P % 16 == 0
    old = pkv.set_decode_split(pkv.PKV_SPLIT_BALANCED)
    try:
        assert pkv.paged_attention_decode_partition_size(64, 40, 2049, 16, 0) == 0
        assert pkv.paged_attention_decode_partition_size(4096, 8, 2049, 16, 0) > 0  # B > 2048
    finally:
        pkv.set_decode_split(old)
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attention_decode_partition_size(8, 8, 100, 16, 24)  # not a multiple of 16
    # fixed-length partitions: one partition needs no workspace
    assert pkv.paged_attention_decode_workspace_size(8, 64, 8, 128, 1000, 16, 1024) == 0
    # the size covers the balanced split too: counters + one partial slot per unit and per
    # worker (1184 workers)
    slots = 4 * 4 + 1184
    ws = pkv.paged_attention_decode_workspace_size(4, 4, 4, 64, 34, 16, 0)
    assert slots * (64 + 2) * 4 <= ws <= slots * (64 + 2) * 4 + 1024
    assert pkv.paged_attention_decode_workspace_size(0, 4, 4, 64, 34, 16, 0) == 0
    # split partitions: counters + (max, sum) + D floats per (b, kvh, part, head)
    ws = pkv.paged_attention_decode_workspace_size(8, 64, 8, 128, 131073, 16, 2048)
    parts = -(-131073 // 2048)
    assert ws >= 8 * 8 * parts * 8 * (128 + 2) * 4
    assert ws <= 8 * 8 * parts * 8 * (128 + 2) * 4 + 4096
    assert pkv.paged_attention_decode_workspace_size(8, 63, 8, 128, 1000, 16, 0) == 0  # invalid


def _decode(lib, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, mb=8, sl=FAKE, msl=100, B=2, Hq=8, Hkv=2,
             D=128, bs=16, nb=64, scale=0.1, dt=0, part=0, ws=None, wsb=0)
    a.update(kw)
    return lib.paged_attention_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["mb"], a["sl"],
                                      a["msl"], a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"],
                                      a["nb"], a["scale"], a["dt"], a["part"], a["ws"], a["wsb"],
                                      None)


@host_only
def test_decode_rejects_bad_arguments(lib):
    assert _decode(lib, out=None) == ERR_ARG
    assert _decode(lib, q=FAKE + 8) == ERR_ARG  # misaligned
    assert _decode(lib, Hq=7) == ERR_ARG  # Hq % Hkv != 0
    assert _decode(lib, Hkv=0) == ERR_ARG
    assert _decode(lib, dt=7) == ERR_ARG
    assert _decode(lib, scale=float("nan")) == ERR_ARG
    assert _decode(lib, part=24) == ERR_ARG
    assert _decode(lib, D=96) == ERR_UNSUP
    assert _decode(lib, D=256, dt=1) == ERR_UNSUP
    assert _decode(lib, bs=24) == ERR_UNSUP  # 8, or a multiple of 16
    assert _decode(lib, bs=4) == ERR_UNSUP
    assert _decode(lib, Hq=64, Hkv=2) == ERR_UNSUP  # G = 32
    assert _decode(lib, msl=8 * 16 + 1) == ERR_RANGE
    assert _decode(lib, nb=(1 << 31) // 16) == ERR_RANGE
    # needs a workspace (split into partitions)
    assert _decode(lib, msl=128, part=16) == ERR_WS
    assert _decode(lib, msl=128, part=16, ws=FAKE, wsb=16) == ERR_WS
    assert _decode(lib, msl=128, part=16, ws=FAKE + 16, wsb=1 << 20) == ERR_WS  # misaligned
    # an empty batch is a no-op that succeeds without touching the device
    assert _decode(lib, B=0) == 0


@host_only
def test_contiguous_control_rejects_bad_arguments(lib):
    def c(**kw):
        a = dict(out=FAKE, k=FAKE, msl=100, stride=128, B=2, Hq=8, Hkv=2, D=128, dt=0, part=0)
        a.update(kw)
        return lib.paged_attention_decode_contiguous(
            a["out"], FAKE, a["k"], FAKE, FAKE, a["msl"], a["stride"], a["B"], a["Hq"], a["Hkv"],
            a["D"], 0.1, a["dt"], a["part"], None, 0, None)
    assert c(stride=99) == ERR_ARG  # a row stride shorter than the longest sequence
    assert c(stride=0) == ERR_ARG
    assert c(out=None) == ERR_ARG
    assert c(k=FAKE + 8) == ERR_ARG
    assert c(dt=1) == ERR_UNSUP  # the control runs the bf16 tensor-core kernel only
    assert c(D=96) == ERR_UNSUP
    assert c(msl=128, part=16) == ERR_WS  # split into partitions without a workspace
    assert c(B=0) == 0


@host_only
def test_write_and_copy_reject_bad_arguments(lib):
    w = lambda **kw: lib.paged_kv_write(kw.get("k", FAKE), FAKE, FAKE, FAKE, kw.get("slots", FAKE),
                                        kw.get("N", 4), kw.get("Hkv", 8), kw.get("D", 128), 16,
                                        kw.get("nb", 64), kw.get("dt", 0), None)
    assert w(k=None) == ERR_ARG
    assert w(k=FAKE + 4) == ERR_ARG
    assert w(slots=FAKE + 4) == ERR_ARG
    assert w(N=-1) == ERR_ARG
    assert w(dt=3) == ERR_ARG
    assert w(Hkv=1, D=3) == ERR_UNSUP  # row of 6 bytes
    assert w(N=0) == 0
    c = lambda **kw: lib.copy_blocks(kw.get("k", FAKE), FAKE, kw.get("m", FAKE), kw.get("P", 3),
                                     kw.get("bb", 32768), kw.get("nb", 64), None)
    assert c(k=None) == ERR_ARG
    assert c(m=FAKE + 4) == ERR_ARG
    assert c(bb=24) == ERR_UNSUP
    assert c(P=-1) == ERR_ARG
    assert c(nb=0) == ERR_ARG
    assert c(P=0) == 0


def test_decode_split_selector(lib):
    old = pkv.set_decode_split(pkv.PKV_SPLIT_BALANCED)
    assert pkv.set_decode_split(old) == pkv.PKV_SPLIT_BALANCED
    with pytest.raises(pkv.PagedKVError):
        pkv.set_decode_split(5)


def test_decode_cta_selector(lib):
    old = pkv.set_decode_ctas(7)
    assert pkv.set_decode_ctas(old) == 7
    with pytest.raises(pkv.PagedKVError):
        pkv.set_decode_ctas(-1)


def test_launch_overlap_switch(lib):
    old = pkv.set_launch_overlap(False)
    assert pkv.set_launch_overlap(True) is False
    assert pkv.set_launch_overlap(old) is True
    assert lib.pkv_set_launch_overlap(2) == ERR_ARG


def test_decode_path_selector(lib):
    old = pkv.set_decode_path(pkv.PKV_PATH_TENSOR_CORES)
    assert pkv.set_decode_path(pkv.PKV_PATH_CUDA_CORES) == pkv.PKV_PATH_TENSOR_CORES
    assert pkv.set_decode_path(old) == pkv.PKV_PATH_CUDA_CORES
    with pytest.raises(pkv.PagedKVError):
        pkv.set_decode_path(9)


def _prefill(lib, **kw):
    a = dict(out=FAKE, q=FAKE, bt=FAKE, mb=8, sl=FAKE, cu=FAKE, T=64, mq=32, msl=128, B=2, Hq=32,
             Hkv=8, D=128, bs=16, nb=64, scale=0.088, dt=0, ws=None, wsb=0)
    a.update(kw)
    return lib.paged_attention_prefill(a["out"], a["q"], FAKE, FAKE, a["bt"], a["mb"], a["sl"],
                                       a["cu"], a["T"], a["mq"], a["msl"], a["B"], a["Hq"],
                                       a["Hkv"], a["D"], a["bs"], a["nb"], a["scale"], a["dt"],
                                       a["ws"], a["wsb"], None)


def test_prefill_workspace_size(lib):
    # two query tiles of 128 / G tokens per work item: G = 4 -> 64 tokens per item
    assert lib.paged_attention_prefill_workspace_size(2, 32, 8, 100) == (2 + 2 * 2 * 8) * 4
    assert lib.paged_attention_prefill_workspace_size(3, 8, 8, 512) == (2 + 3 * 2 * 8) * 4
    assert lib.paged_attention_prefill_workspace_size(0, 32, 8, 100) == 0
    assert lib.paged_attention_prefill_workspace_size(2, 30, 8, 100) == 0  # Hq % Hkv != 0
    assert lib.paged_attention_prefill_workspace_size(2, 32, 8, 0) == 0


@host_only
def test_prefill_rejects_bad_arguments(lib):
    assert _prefill(lib, out=None) == ERR_ARG
    assert _prefill(lib, q=FAKE + 8) == ERR_ARG  # misaligned
    assert _prefill(lib, sl=FAKE + 2) == ERR_ARG
    assert _prefill(lib, Hq=30) == ERR_ARG  # Hq % Hkv != 0
    assert _prefill(lib, scale=float("inf")) == ERR_ARG
    assert _prefill(lib, dt=1) == ERR_UNSUP  # fp32 has no tensor-core path here
    assert _prefill(lib, D=96) == ERR_UNSUP
    assert _prefill(lib, Hq=256, Hkv=8) == ERR_UNSUP  # G = 32
    assert _prefill(lib, bs=8) == ERR_UNSUP
    assert _prefill(lib, mq=0) == ERR_RANGE
    assert _prefill(lib, mq=200) == ERR_RANGE  # longer than max_seq_len
    assert _prefill(lib, msl=8 * 16 + 1) == ERR_RANGE  # more than the table holds
    n = lib.paged_attention_prefill_workspace_size(2, 32, 8, 32)
    assert _prefill(lib, ws=FAKE + 2, wsb=n) == ERR_ARG  # misaligned workspace
    assert _prefill(lib, ws=FAKE, wsb=n - 4) == ERR_ARG  # too small
    # empty calls succeed without touching the device
    assert _prefill(lib, B=0) == 0
    assert _prefill(lib, T=0) == 0


def test_prefill_path_selector(lib):
    old = pkv.set_prefill_path(pkv.PKV_PREFILL_SINGLE_TILE)
    assert pkv.set_prefill_path(old) == pkv.PKV_PREFILL_SINGLE_TILE
    with pytest.raises(pkv.PagedKVError):
        pkv.set_prefill_path(4)
