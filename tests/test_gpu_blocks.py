"""Block copy (copy-on-write) on the GPU, and the pages' sharing scenario end to
end: a prompt written once, forked, branches that diverge (copy-on-write of the
shared partial block), then decode of every branch against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, to_f64
from paged_kv_cache_432_b200 import build as pa_build
from paged_kv_cache_432_b200 import pagedattn as pa
from paged_kv_cache_432_b200 import workload as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _clean():
    if torch.cuda.is_available():
        pa_build.build()
        pa.device_error(clear=True)
    yield


def _bits(a):
    return a.view(np.uint32) if a.dtype == np.float32 else a


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("Hkv,D", [(32, 128), (2, 64), (8, 128)])
def test_copy_blocks_bit_exact(dtype, Hkv, D):
    g = torch.Generator(device=DEV).manual_seed(Hkv + D)
    NB = 40
    kc = torch.randn((NB, Hkv, 16, D), generator=g, device=DEV).to(dtype)
    vc = torch.randn((NB, Hkv, 16, D), generator=g, device=DEV).to(dtype)
    src = [1, 5, 9, 33, 2, 3]
    dst = [20, 21, 39, 0, 7, NB + 2]  # the last pair points outside the pool
    hk, hv = wl.as_numpy(kc), wl.as_numpy(vc)
    pa.copy_blocks(kc, vc, torch.tensor(src, dtype=torch.int32, device=DEV),
                   torch.tensor(dst, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    ek, ev, bad = oracle.copy_blocks(hk, hv, src, dst)
    assert bad == 1
    assert np.array_equal(_bits(wl.as_numpy(kc)), _bits(ek))
    assert np.array_equal(_bits(wl.as_numpy(vc)), _bits(ev))
    assert pa.device_error() == pa.PA_DEVERR_BLOCK_OOB


def test_fork_diverge_copy_on_write_then_decode():
    Hq, Hkv, D, NB = 8, 2, 128, 64
    gen = torch.Generator().manual_seed(11)
    bm = pa.BlockManager(NB, 16, 32)
    nan = float("nan")
    kc = torch.full((NB, Hkv, 16, D), nan, dtype=torch.bfloat16, device=DEV)
    vc = torch.full_like(kc, nan)
    hk, hv = wl.as_numpy(kc), wl.as_numpy(vc)  # host mirror, updated by the oracle
    truth = {}

    def write(seq, n):
        nonlocal hk, hv
        slots, copies = bm.append(seq, n)
        if copies:
            src = torch.tensor([c[0] for c in copies], dtype=torch.int32, device=DEV)
            dst = torch.tensor([c[1] for c in copies], dtype=torch.int32, device=DEV)
            pa.copy_blocks(kc, vc, src, dst)
            hk, hv, _ = oracle.copy_blocks(hk, hv, src.cpu().numpy(), dst.cpu().numpy())
        K = torch.randn((n, Hkv, D), generator=gen).to(torch.bfloat16)
        V = torch.randn((n, Hkv, D), generator=gen).to(torch.bfloat16)
        sl = torch.tensor(slots, dtype=torch.int64)
        pa.cache_write(K.to(DEV), V.to(DEV), sl.to(DEV), kc, vc)
        hk, hv, _ = oracle.cache_write(wl.as_numpy(K), wl.as_numpy(V), sl.numpy(), hk, hv)
        tk, tv = truth.get(seq, (np.zeros((0, Hkv, D), np.uint16), np.zeros((0, Hkv, D), np.uint16)))
        truth[seq] = (np.concatenate([tk, wl.as_numpy(K)]), np.concatenate([tv, wl.as_numpy(V)]))
        return copies

    bm.add(0)
    assert write(0, 35) == []                    # the prompt: 3 blocks, 13 free slots in the last
    for child in (1, 2):
        bm.fork(0, child)
        truth[child] = truth[0]
    assert len(write(1, 1)) == 1                  # diverges inside the shared partial block
    assert len(write(2, 20)) == 1
    assert write(0, 5) == []                      # the prompt is the last holder of its block now
    bm.fork(2, 3)
    truth[3] = truth[2]
    assert len(write(3, 12)) == 1
    write(1, 40)
    torch.cuda.synchronize()
    # the device pools are exactly what the oracle's copies and writes produce
    assert np.array_equal(wl.as_numpy(kc), hk) and np.array_equal(wl.as_numpy(vc), hv)

    seqs = [0, 1, 2, 3]
    tab, lens = bm.tables(seqs, 8)
    q = torch.randn((len(seqs), Hq, D), generator=gen).to(torch.bfloat16)
    scale = wl.scale_for(D)
    out = pa.decode(q.to(DEV), kc, vc, tab.to(DEV), lens.to(DEV), scale, max_seq_len=int(lens.max()))
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    # expected: every branch's own tokens in a fresh private pool
    nbs = [-(-int(L) // 16) for L in lens]
    pk = np.zeros((sum(nbs), Hkv, 16, D), np.uint16)
    pv = np.zeros_like(pk)
    ptab = np.full((len(seqs), max(nbs)), -1, np.int32)
    base = 0
    for i, s in enumerate(seqs):
        L = int(lens[i])
        assert truth[s][0].shape[0] == L
        ptab[i, : nbs[i]] = np.arange(base, base + nbs[i])
        slots = np.array([(base + t // 16) * 16 + t % 16 for t in range(L)], np.int64)
        pk, pv, _ = oracle.cache_write(truth[s][0], truth[s][1], slots, pk, pv)
        base += nbs[i]
    ref = oracle.paged_decode(wl.as_numpy(q), pk, pv, ptab, lens.numpy(), scale)
    assert_close(to_f64(out), ref, torch.bfloat16, "branches after copy-on-write")
    assert pa.device_error() == 0
