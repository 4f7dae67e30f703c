"""The C-ABI library loads, exports every symbol its header declares, and its
host-side logic (sizing, validation) behaves as documented.  No compute calls:
nothing here needs a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from paged_kv_cache_432_b200 import build as pa_build
from paged_kv_cache_432_b200 import pagedattn as pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedattn.h")


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return pa.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["pa_cache_write", "pa_decode", "pa_decode_partitions", "pa_decode_reduce",
              "pa_decode_workspace_size", "pa_decode_partition_blocks", "pa_get_device_error",
              "pa_status_string"]:
        assert n in names
    assert set(names) == set(pa.SIGNATURES), "binding and header disagree"


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (pa_[a-z0-9_]+)\b", out))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(lib, n)
    # nothing else of ours leaks out of the library
    assert exported == set(declared_functions())


def test_status_strings(lib):
    assert lib.pa_status_string(pa.PA_OK) == b"ok"
    for s in (pa.PA_ERR_INVALID_ARG, pa.PA_ERR_UNSUPPORTED, pa.PA_ERR_WORKSPACE, pa.PA_ERR_CUDA):
        assert len(lib.pa_status_string(s)) > 5


def test_partition_policy(lib):
    assert pa.partition_blocks(8, 8, 131072, 32) == 32
    assert pa.partition_blocks(8, 8, 131072, -1) >= 131072 // 16
    assert pa.partition_blocks(8, 8, 512, 0) == 0           # auto: the balanced split
    assert pa.partition_blocks(64, 32, 2048, 0) == 0
    assert lib.pa_decode_partition_blocks(8, 8, 100, 8, 0) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_partition_blocks(8, 8, 100, 16, -2) == pa.PA_ERR_INVALID_ARG


def test_workspace_size_matches_documented_layout(lib):
    a256 = lambda x: (x + 255) // 256 * 256

    def layout(N, Hq, Hkv, D, P):
        rows = N * Hq
        return 2 * a256(rows * P * 4) + a256(rows * P * D * 4) + a256(N * Hkv * 4)

    N, Hq, Hkv, D, L = 8, 64, 8, 128, 131072
    nb = L // 16
    assert pa.workspace_size(N, Hq, Hkv, D, L, 32) == layout(N, Hq, Hkv, D, -(-nb // 32))
    assert pa.workspace_size(N, Hq, Hkv, D, 512, 32) == 0        # one partition: no workspace
    assert pa.workspace_size(N, Hq, Hkv, D, L, -1) == 0
    assert pa.workspace_size(N, Hq, Hkv, D, 513, 32) == layout(N, Hq, Hkv, D, 2)
    # balanced split: a unit of nb blocks meets at most ceil(nb / 16) + 1 warp ranges
    assert pa.workspace_size(N, Hq, Hkv, D, L, 0) == layout(N, Hq, Hkv, D, -(-nb // 16) + 1)
    assert pa.workspace_size(N, Hq, Hkv, D, 100, 0) == layout(N, Hq, Hkv, D, 2)
    assert pa.workspace_size(N, Hq, Hkv, D, 0, 0) == 0


def test_shared_prefix_workspace_size(lib):
    a256 = lambda x: (x + 255) // 256 * 256
    N, Hq, Hkv, D = 128, 32, 8, 128
    # 16 reserved key-split slots for the prefix, then the private part:
    # (4604 - 4096) tokens -> 32 blocks -> balanced bound ceil(32/16)+1 = 3 pieces
    P = 16 + 3
    rows = N * Hq
    # + 256 bytes: the tile kernel's item counter
    expect = 2 * a256(rows * P * 4) + a256(rows * P * D * 4) + a256(N * Hkv * 4) + 256
    assert lib.pa_decode_shared_prefix_workspace_size(N, Hq, Hkv, D, 4604, 256, 16, 0) == expect
    # several prompt groups: the private part can be a whole sequence (4604 tokens -> 288 blocks ->
    # ceil(288/16)+1 = 19 pieces) after the 16 slots
    P = 16 + 19
    expect = 2 * a256(rows * P * 4) + a256(rows * P * D * 4) + a256(N * Hkv * 4) + 256
    assert lib.pa_decode_shared_prefix_groups_workspace_size(N, Hq, Hkv, D, 4604, 256, 4, 16, 0) == expect
    # no shared blocks: the plain decode's size
    assert lib.pa_decode_shared_prefix_workspace_size(N, Hq, Hkv, D, 4604, 0, 16, 0) == \
        lib.pa_decode_workspace_size(N, Hq, Hkv, D, 4604, 16, 0)
    # a prefix longer than the longest sequence is rejected
    assert lib.pa_decode_shared_prefix_workspace_size(N, Hq, Hkv, D, 1000, 256, 16, 0) == 0


def _tile_splits(sms, work_tiles, nb_max):
    """The key chunking the tile kernel picks (as documented in the header):
    as many chunks as fill the SMs, or, for long units, up to 16 items per SM
    with chunks of at least 256 blocks; at most 16, in multiples of 4 blocks."""
    nb_max = max(1, nb_max)
    want = max(1, sms // work_tiles if work_tiles else 1)
    if work_tiles:
        want = max(want, min(-(-16 * sms // work_tiles), nb_max // 256))
    want = min(16, want)
    ch = -(-nb_max // want)
    ch = -(-ch // 4) * 4
    return -(-nb_max // ch)


def test_multi_query_workspace_and_limits(lib):
    import torch

    a256 = lambda x: (x + 255) // 256 * 256
    N, T, Hq, Hkv, D, L = 4, 13, 8, 2, 128, 3000
    layout = lambda P: 2 * a256(T * Hq * P * 4) + a256(T * Hq * P * D * 4) + a256(N * Hkv * 4)
    P = -(-(-(-L // 16)) // 16) + 1  # balanced bound of the warp-level path
    # the tile path (group x query tokens > 16) keeps one partial per key chunk
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 1 << 30
    tiles = -(-T // (2 * (128 // (Hq // Hkv)))) + N  # tiles of two 128-row halves
    C = _tile_splits(sms, tiles * Hkv, -(-L // 16))
    want = max(layout(P), (layout(C) if C > 1 else 0) + 256)  # + the tile kernel's item counter
    assert lib.pa_decode_multi_workspace_size(N, T, Hq, Hkv, D, L, 16, 0) == want
    # fp32 or a missing q_start are refused before anything is launched
    assert lib.pa_decode_multi(16, 16, T, 5, 16, 16, 16, 64, 16, L, N, 8, 2, D, 64, 16, 0.1, 0, None, 0, 16,
                               pa.PA_DTYPE_F32, None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_multi(16, 16, T, 2, 16, 16, 16, 64, 16, L, N, 8, 2, D, 64, 16, 0.1, 0, None, 0, 16,
                               pa.PA_DTYPE_F32, None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_multi(16, None, T, 2, 16, 16, 16, 64, 16, L, N, 8, 2, D, 64, 16, 0.1, 0, None, 0, 16,
                               pa.PA_DTYPE_BF16, None) == pa.PA_ERR_INVALID_ARG


def _decode_rc(lib, **over):
    args = dict(q=16, k=16, v=16, bt=16, mb=4, sl=16, msl=64, N=2, Hq=4, Hkv=2, D=128, NB=8, B=16,
                scale=0.1, pb=0, ws=None, wsb=0, out=16, dt=pa.PA_DTYPE_BF16)
    args.update(over)
    a = args
    return lib.pa_decode(a["q"], a["k"], a["v"], a["bt"], a["mb"], a["sl"], a["msl"], a["N"], a["Hq"],
                         a["Hkv"], a["D"], a["NB"], a["B"], a["scale"], a["pb"], a["ws"], a["wsb"],
                         a["out"], a["dt"], None)


def test_decode_rejects_bad_arguments_on_the_host(lib):
    # (fake, never dereferenced addresses: validation happens before any CUDA call)
    assert _decode_rc(lib, q=None) == pa.PA_ERR_INVALID_ARG
    assert _decode_rc(lib, q=8) == pa.PA_ERR_INVALID_ARG            # misaligned
    assert _decode_rc(lib, out=None) == pa.PA_ERR_INVALID_ARG
    assert _decode_rc(lib, Hq=3) == pa.PA_ERR_INVALID_ARG           # not a multiple of Hkv
    assert _decode_rc(lib, D=96) == pa.PA_ERR_UNSUPPORTED
    assert _decode_rc(lib, B=32) == pa.PA_ERR_UNSUPPORTED
    assert _decode_rc(lib, dt=7) == pa.PA_ERR_UNSUPPORTED
    assert _decode_rc(lib, Hq=34, Hkv=2) == pa.PA_ERR_UNSUPPORTED   # group of 17
    assert _decode_rc(lib, mb=0) == pa.PA_ERR_INVALID_ARG
    assert _decode_rc(lib, pb=-5) == pa.PA_ERR_INVALID_ARG
    assert _decode_rc(lib, scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    # split needed (1000 tokens, 32-block partitions) but no workspace
    assert _decode_rc(lib, mb=64, msl=1000, pb=32) == pa.PA_ERR_WORKSPACE
    assert _decode_rc(lib, mb=64, msl=1000, pb=32, ws=256, wsb=16) == pa.PA_ERR_WORKSPACE


def test_cache_write_rejects_bad_arguments_on_the_host(lib):
    f = lib.pa_cache_write
    ok = dict(k=16, v=16, s=16, T=4, H=2, D=128, kc=16, vc=16, NB=8, B=16, dt=pa.PA_DTYPE_BF16)

    def rc(**o):
        a = dict(ok, **o)
        return f(a["k"], a["v"], a["s"], a["T"], a["H"], a["D"], a["kc"], a["vc"], a["NB"], a["B"], a["dt"], None)

    assert rc(k=None) == pa.PA_ERR_INVALID_ARG
    assert rc(s=12) == pa.PA_ERR_INVALID_ARG        # slots not 8-byte aligned
    assert rc(kc=24) == pa.PA_ERR_INVALID_ARG
    assert rc(T=-1) == pa.PA_ERR_INVALID_ARG
    assert rc(NB=0) == pa.PA_ERR_INVALID_ARG
    assert rc(D=80) == pa.PA_ERR_UNSUPPORTED
    assert rc(B=8) == pa.PA_ERR_UNSUPPORTED
    assert rc(T=0) == pa.PA_OK                      # nothing to do, nothing launched


def test_fp8_entry_points_reject_bad_arguments_on_the_host(lib):
    f = lib.pa_cache_write_fp8
    ok = dict(k=16, v=16, s=16, T=4, H=2, D=128, kc=16, vc=16, NB=8, B=16, ks=32, vs=32)

    def rc(**o):
        a = dict(ok, **o)
        return f(a["k"], a["v"], a["s"], a["T"], a["H"], a["D"], a["kc"], a["vc"], a["NB"], a["B"], a["ks"],
                 a["vs"], None)

    assert rc(ks=None) == pa.PA_ERR_INVALID_ARG      # inverse scales are required
    assert rc(vs=34) == pa.PA_ERR_INVALID_ARG        # not 4-byte aligned
    assert rc(kc=8) == pa.PA_ERR_INVALID_ARG
    assert rc(D=96) == pa.PA_ERR_UNSUPPORTED
    assert rc(B=32) == pa.PA_ERR_UNSUPPORTED
    assert rc(T=0) == pa.PA_OK

    d = lib.pa_decode_fp8
    base = [16, 16, 16, 32, 32, 16, 4, 16, 64, 2, 8, 2, 128, 8, 16, 0.1, -1, None, 0, 16, None]

    def drc(i=None, val=None):
        a = list(base)
        if i is not None:
            a[i] = val
        return d(*a)

    assert drc(3, None) == pa.PA_ERR_INVALID_ARG     # k_scale
    assert drc(4, None) == pa.PA_ERR_INVALID_ARG     # v_scale
    assert drc(4, 33) == pa.PA_ERR_INVALID_ARG       # misaligned v_scale
    assert drc(0, 8) == pa.PA_ERR_INVALID_ARG        # misaligned q
    assert drc(12, 96) == pa.PA_ERR_UNSUPPORTED      # head_dim
    assert drc(10, 34) == pa.PA_ERR_UNSUPPORTED      # 34 / 2 = group of 17
    assert drc(15, float("inf")) == pa.PA_ERR_INVALID_ARG

    # the partition step alone validates the same way
    dp = lib.pa_decode_fp8_partitions

    def prc(i=None, val=None):
        a = list(base)
        if i is not None:
            a[i] = val
        return dp(*a)

    assert prc(3, None) == pa.PA_ERR_INVALID_ARG
    assert prc(0, 8) == pa.PA_ERR_INVALID_ARG
    assert prc(12, 96) == pa.PA_ERR_UNSUPPORTED
    # the E4M3 merge: sizes as pa_decode_reduce, the workspace checked first
    r = lib.pa_decode_fp8_reduce
    assert r(16, 2048, 4, 8, 2, 128, 128, 16, 0, None, 0, 16, None) == pa.PA_ERR_WORKSPACE
    assert r(16, 2048, 4, 8, 2, 96, 128, 16, 0, 256, 1 << 20, 16, None) == pa.PA_ERR_UNSUPPORTED
    assert r(16, 2048, 4, 8, 3, 128, 128, 16, 0, 256, 1 << 20, 16, None) == pa.PA_ERR_INVALID_ARG


def test_get_device_error_rejects_null(lib):
    assert lib.pa_get_device_error(None, 0, None) == pa.PA_ERR_INVALID_ARG


def _comment_before(name: str) -> str:
    """The comment block that directly precedes the declaration of `name`."""
    src = open(HEADER).read()
    i = re.search(r"PA_API[^;]*?\b" + name + r"\s*\(", src).start()
    j = src.rfind("*/", 0, i)
    return src[src.rfind("/*", 0, j):j]


@pytest.mark.parametrize("name", ["pa_cache_write", "pa_decode", "pa_decode_workspace_size",
                                  "pa_get_device_error", "pa_status_string", "pa_decode_fp8_partitions",
                                  "pa_decode_fp8_reduce"])
def test_boundary_calls_cite_a_passage_or_say_plumbing(name):
    """Each call of the boundary names the page passage that defines it, or
    says that it is interface plumbing with no passage."""
    c = _comment_before(name)
    pages = ("slavadubrov.com", "aiunderstanding.org", "de.news.hada.io", "artificials.ru")
    assert any(p in c for p in pages) or "Interface plumbing" in c, name


def test_prompt_groups_and_prefill_reject_bad_arguments_on_the_host(lib):
    """The prompt-group decode and the prefill path validate on the host
    before any CUDA call (fake, never dereferenced addresses)."""
    g = lib.pa_decode_shared_prefix_groups

    def grc(**over):
        a = dict(q=16, k=16, v=16, bt=16, mb=64, sl=16, msl=1000, gs=16, gb=16, G=2, maxs=32, N=4, Hq=8, Hkv=2,
                 D=128, NB=64, B=16, scale=0.1, pb=0, ws=256, wsb=1 << 30, out=16, dt=pa.PA_DTYPE_BF16)
        a.update(over)
        return g(a["q"], a["k"], a["v"], a["bt"], a["mb"], a["sl"], a["msl"], a["gs"], a["gb"], a["G"], a["maxs"],
                 a["N"], a["Hq"], a["Hkv"], a["D"], a["NB"], a["B"], a["scale"], a["pb"], a["ws"], a["wsb"],
                 a["out"], a["dt"], None)

    assert grc(gs=None) == pa.PA_ERR_INVALID_ARG
    assert grc(gb=None) == pa.PA_ERR_INVALID_ARG
    assert grc(gs=18) == pa.PA_ERR_INVALID_ARG          # misaligned
    assert grc(G=0) == pa.PA_ERR_INVALID_ARG
    assert grc(maxs=-1) == pa.PA_ERR_INVALID_ARG
    assert grc(maxs=100) == pa.PA_ERR_INVALID_ARG       # more shared blocks than max_seq_len holds
    assert grc(dt=pa.PA_DTYPE_F32) == pa.PA_ERR_UNSUPPORTED
    need = lib.pa_decode_shared_prefix_groups_workspace_size(4, 8, 2, 128, 1000, 32, 2, 16, 0)
    assert need > 0
    assert grc(wsb=need - 1) == pa.PA_ERR_WORKSPACE
    assert grc(ws=None) == pa.PA_ERR_WORKSPACE
    # the prefill path (group 4 x 64 query tokens > 16 rows): the workspace holds at least its counter
    m = lib.pa_decode_multi
    assert m(16, 16, 64, 64, 16, 16, 16, 64, 16, 1000, 1, 8, 2, 128, 64, 16, 0.1, 0, None, 0, 16,
             pa.PA_DTYPE_BF16, None) == pa.PA_ERR_WORKSPACE
    assert m(16, 16, 64, 64, 16, 16, 16, 64, 16, 1000, 1, 8, 2, 96, 64, 16, 0.1, 0, 256, 1 << 20, 16,
             pa.PA_DTYPE_BF16, None) == pa.PA_ERR_UNSUPPORTED  # head_dim 96
