"""Paged chunked prefill (tcgen05 tensor cores) vs the fp64 oracle (needs a B200).

Same tolerance as decode: |gpu - ref| <= 2e-3 + 1e-2 |ref|.  Cases span
several 128-row query tiles, ragged last tiles, GQA groups 1 / 4 / 8 / 16,
8- and 16-token blocks, prefixes that end inside a block, and chunks that are
the whole sequence.
"""
import numpy as np
import pytest
import torch

from paged_helpers import assert_close, device_inputs, oracle_subset
from workloads import make_workload

pytestmark = pytest.mark.gpu

pkv = pytest.importorskip("paged_kv_cache_371_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    pkv.device_error(reset=True)
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("Hq,Hkv,bs,q_len,lens", [
    (8, 8, 16, 37, [37, 100]),            # MHA rows, whole-sequence chunk and a prefix
    (32, 8, 16, 64, [64, 200, 1031]),     # G=4: 16 positions per tile, 4 tiles
    (64, 8, 16, 48, [300, 48, 777]),      # G=8: 16 positions per tile, ragged last tile
    (16, 1, 8, 24, [24, 95, 513]),        # G=16, 8-token blocks
    (8, 8, 8, 200, [200, 333]),           # MHA, 2 tiles of 128 positions
])
def test_prefill_full_compare(Hq, Hkv, bs, q_len, lens):
    wl = make_workload("llama70b_gqa", "cuda", lens=np.array(lens, np.int32), bs=bs, q_len=q_len,
                       Hq=Hq, Hkv=Hkv, D=128, seed=q_len + Hq)
    bt, cl = device_inputs(wl)
    out = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = oracle_subset(wl, list(range(wl.B)), q_len=q_len)
    assert_close(out, ref, f"prefill Hq{Hq} Hkv{Hkv} bs{bs} q{q_len}")


def test_prefill_matches_verify_for_short_windows():
    """A 5-token window through prefill and through the verify path agree."""
    wl = make_workload("long_verify", "cuda", B=2, max_len=3000)
    bt, cl = device_inputs(wl)
    a = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, 5)
    b = pkv.paged_verify_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, 5)
    ref = oracle_subset(wl, [0, 1], q_len=5)
    assert_close(a, ref, "prefill")
    assert_close(b, ref, "verify")
