"""The serving flow end to end on the GPU: requests are admitted through the
native block manager (shared prompt prefixes hit its cache), the uncached part
of each prompt is prefilled in chunks -- several sequences per call, mixed
with decode requests of sequences already generating -- and then every
sequence generates through batched appends and decode steps. Every output row
is compared with the oracle's causal attention over that sequence's own K/V
laid out privately (no sharing, no paging of its own).

The K/V row of a position is a seeded function of the token prefix through
it, so equal prefixes have equal K/V -- what makes reusing cached blocks valid.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import compare
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200.blocks import BlockManager
from test_gpu_block_manager import Model

pytestmark = pytest.mark.gpu

NKV, NQ, D = 8, 32, 128


def oracle_rows(model, entries, q, bs):
    """fp64 attention of chunk rows: entries = [(seq, first position, n rows)]
    in the order of q's rows, each row attending causally over its sequence's
    private K/V."""
    nblk = sum(-(-(len(model.toks[s])) // bs) for s, _, _ in entries)
    kp = O.new_pool(nblk, NKV, bs, D, False, 0x7FC0)
    vp = O.new_pool(nblk, NKV, bs, D, False, 0x7FC0)
    maxb = max(-(-(p0 + n) // bs) for _, p0, n in entries)
    tables = np.full((len(entries), maxb), -1, np.int32)
    cu, ctx = [0], []
    base = 0
    for r, (s, p0, n) in enumerate(entries):
        L = p0 + n  # the rows see positions < p0 + n
        nb = -(-L // bs)
        tables[r, :nb] = np.arange(base, base + nb)
        slots = torch.arange(base * bs, base * bs + L, dtype=torch.int32)
        assert O.store_kvcache(torch.stack(model.k[s][:L]), torch.stack(model.v[s][:L]), kp, vp, slots, nblk, bs) == 0
        base += nb
        cu.append(cu[-1] + n)
        ctx.append(L)
    out, st = O.paged_attention_prefill(q.cpu(), kp, vp, tables, np.array(cu, np.int32), np.array(ctx, np.int32),
                                        NKV, bs, 1.0 / math.sqrt(D), num_threads=8)
    assert st == O.ORC_OK
    return out


@pytest.mark.parametrize("bs", [16, 256])
def test_admit_prefill_in_chunks_then_decode(bs):
    dev = "cuda"
    rng = np.random.default_rng(21)
    num_blocks = 4096 if bs == 16 else 320
    bm = BlockManager(num_blocks, bs)
    model = Model()
    kp = torch.zeros((num_blocks, NKV, bs, D), dtype=torch.bfloat16, device=dev)
    vp = torch.zeros_like(kp)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    chunk = 384

    prompts = [rng.integers(0, 32000, n).tolist() for n in (1200, 700)]
    pending = {}  # seq -> next prompt position still to prefill
    prompt_of = {}
    hits = 0

    def admit(sid, toks):
        nonlocal hits
        st, cached = bm.add_sequence(sid, toks)
        assert st == K.PKV_OK
        model.extend(sid, toks)  # the K/V rows every position will hold
        pending[sid] = cached  # cached blocks already hold their rows: nothing to write for them
        prompt_of[sid] = len(toks)
        hits += cached

    decoding = []

    def run_round(tag):
        entries, k_rows, v_rows, slots = [], [], [], []
        for sid in sorted(pending):  # prefill chunks
            p0 = pending[sid]
            n = min(chunk, prompt_of[sid] - p0)
            entries.append((sid, p0, n))
            slots += bm.slots(sid, p0, n)
            k_rows += model.k[sid][p0:p0 + n]
            v_rows += model.v[sid][p0:p0 + n]
        for sid in decoding:  # one new token each
            t = int(rng.integers(0, 32000))
            k, v = model.extend(sid, [t])
            st, slot = bm.append_token(sid, t)
            assert st == K.PKV_OK
            entries.append((sid, len(model.toks[sid]) - 1, 1))
            slots.append(slot)
            k_rows.append(k[0])
            v_rows.append(v[0])
        K.store_kvcache(torch.stack(k_rows).to(dev), torch.stack(v_rows).to(dev), kp, vp,
                        torch.tensor(slots, dtype=torch.int32, device=dev), dev_err=err)
        ids = [s for s, _, _ in entries]
        maxb = max(-(-len(model.toks[s]) // bs) for s in ids)
        tables, _ = bm.block_tables(ids, maxb)
        # a chunk's context ends at its last row (the rest of the prompt is not attended yet)
        ctx = np.array([p0 + n for _, p0, n in entries], np.int32)
        cu = np.concatenate([[0], np.cumsum([n for _, _, n in entries])]).astype(np.int32)
        q = torch.from_numpy(rng.standard_normal((int(cu[-1]), NQ, D), dtype=np.float32)).to(torch.bfloat16)
        out = K.paged_attention_prefill(q.to(dev), kp, vp, torch.from_numpy(tables).to(dev),
                                        torch.from_numpy(cu).to(dev), torch.from_numpy(ctx).to(dev), scale,
                                        int(max(n for _, _, n in entries)), dev_err=err)
        assert K.read_device_error(err) == K.PKV_OK
        compare(out, oracle_rows(model, entries, q, bs), False, tag)
        for sid, p0, n in entries:
            if sid in pending:
                pending[sid] = p0 + n
                if pending[sid] == prompt_of[sid]:
                    del pending[sid]
                    decoding.append(sid)

    # wave 1: two different prompts, prefilled in chunks until both generate
    for sid in range(2):
        admit(sid, prompts[sid] + rng.integers(0, 32000, 37).tolist())
    r = 0
    while pending:
        r += 1
        run_round(f"wave 1 round {r}")
    # wave 2: requests sharing those prompts' prefixes hit their (now stored)
    # blocks; their chunks share calls with the first two sequences' decoding
    for sid in range(2, 6):
        p = prompts[sid % 2][: len(prompts[sid % 2]) - int(rng.integers(0, 300))]
        admit(sid, p + rng.integers(0, 32000, int(rng.integers(1, 200))).tolist())
    assert hits > 0, "later requests must hit the cached prefix"
    r = 0
    while pending or r < 2:
        r += 1
        run_round(f"wave 2 round {r}")
    # pure decode steps through the decode kernel on the same pools
    for _ in range(3):
        new = rng.integers(0, 32000, len(decoding)).tolist()
        slots = bm.append_tokens(decoding, new)
        ks, vs = zip(*(model.extend(s, [t]) for s, t in zip(decoding, new)))
        K.store_kvcache(torch.cat(ks).to(dev), torch.cat(vs).to(dev), kp, vp, torch.from_numpy(slots).to(dev),
                        dev_err=err)
        maxb = max(-(-len(model.toks[s]) // bs) for s in decoding)
        tables, lens = bm.block_tables(decoding, maxb)
        q = torch.from_numpy(rng.standard_normal((len(decoding), NQ, D), dtype=np.float32)).to(torch.bfloat16)
        out = K.paged_attention_decode(q.to(dev), kp, vp, torch.from_numpy(tables).to(dev),
                                       torch.from_numpy(lens).to(dev), scale, dev_err=err)
        assert K.read_device_error(err) == K.PKV_OK
        entries = [(s, len(model.toks[s]) - 1, 1) for s in decoding]
        compare(out, oracle_rows(model, entries, q, bs), False, "decode")
