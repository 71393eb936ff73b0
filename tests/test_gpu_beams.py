"""GPU: many-beam search steps (fork / reorder, batched copy-on-write, append,
attention) with the pools kept bit-exact against an oracle mirror and the
attention within tolerance of the oracle."""
import numpy as np
import pytest
import torch

import oracle
from paged_helpers import assert_close
from workloads import normal_fp16

import paged_kv_cache_371_b200 as pkv

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.cpu().numpy().view(np.uint16)


def test_beam_search_steps_bit_exact_pools_and_attention():
    S, W, steps = 16, 8, 6                    # 16 prompts x 8 beams = 128 beams
    Hq, Hkv, D, bs = 32, 8, 128, 16
    rng = np.random.Generator(np.random.PCG64(77))
    prompt = rng.integers(100, 400, size=S)   # ragged: partial last blocks
    nb = int(sum(-(-p // bs) for p in prompt)) + S * W * (steps + 2) + 64
    cap = int(prompt.max()) // bs + steps + 3
    pool = pkv.KVPool(nb, bs, Hkv, D)
    k = normal_fp16((nb, Hkv, bs, D), 1, "cuda")
    v = normal_fp16((nb, Hkv, bs, D), 2, "cuda")
    Kh, Vh = k.cpu().numpy(), v.cpu().numpy()
    tables = np.full((S, cap), -1, np.int32)
    nblk = np.zeros(S, np.int32)
    for s in range(S):
        ids = pool.alloc(-(-int(prompt[s]) // bs))
        tables[s, :len(ids)] = ids
        nblk[s] = len(ids)
    parents = np.repeat(np.arange(S), W).astype(np.int32)
    beam_len = prompt.astype(np.int32)
    total_pairs = 0
    for step in range(steps):
        tables, nblk = pool.beam_reorder(tables, nblk, parents)
        lens = beam_len[parents].astype(np.int32)
        slots, pairs = pool.reserve_slots(tables, nblk, lens)
        total_pairs += len(pairs)
        kn = normal_fp16((S * W, Hkv, D), 10 + step, "cuda")
        vn = normal_fp16((S * W, Hkv, D), 20 + step, "cuda")
        if len(pairs):
            pkv.paged_kv_copy_blocks(k, v, torch.as_tensor(pairs, device="cuda"))
            Kh, Vh = oracle.copy_blocks(Kh, Vh, pairs)
        pkv.paged_kv_append(kn, vn, torch.as_tensor(slots, device="cuda"), k, v)
        Kh, Vh = oracle.append(Kh, Vh, kn.cpu().numpy(), vn.cpu().numpy(), slots)
        assert pkv.device_error() == 0
        assert np.array_equal(_u16(k), Kh.view(np.uint16)), f"K pool differs at step {step}"
        assert np.array_equal(_u16(v), Vh.view(np.uint16)), f"V pool differs at step {step}"
        beam_len = lens + 1
        parents = np.concatenate([g * W + rng.integers(0, W, size=W) for g in range(S)]).astype(np.int32)
    # prompts ending mid-block copy on the first step: every beam but the last writer
    assert total_pairs >= sum((W - 1) for p in prompt if p % bs)
    q = normal_fp16((S * W, 1, Hq, D), 99, "cuda")
    out = pkv.paged_decode_attention(q, k, v, torch.as_tensor(tables, device="cuda"),
                                     torch.as_tensor(beam_len, device="cuda"), D ** -0.5)
    torch.cuda.synchronize()
    ref = oracle.paged_attention(q.cpu().numpy(), Kh, Vh, tables, beam_len, scale=D ** -0.5)
    assert_close(out, ref, "beams")
