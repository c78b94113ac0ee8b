"""The block manager feeding the kernels (B200): requests with shared
prefixes are admitted through the native manager, only their uncached tokens
are written with store_kvcache at the manager's slots, decode steps append
through the batch call and read the manager's block tables; the output must
equal the oracle's attention over each sequence's own logical K/V laid out
privately (no sharing) in a host pool.

The K/V row of position p is a seeded function of the token prefix through p,
so equal prefixes have equal K/V -- what makes reusing cached blocks valid.
"""

import math
import zlib

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import BF16_ABS, compare
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200.blocks import BlockManager

pytestmark = pytest.mark.gpu

NKV, NQ, D, BS = 8, 32, 128, 16


class Model:
    """Per-sequence token streams and the K/V rows their prefixes define."""

    def __init__(self):
        self.toks, self.k, self.v, self.h = {}, {}, {}, {}

    def _rows(self, h):
        r = np.random.default_rng(h).standard_normal((2, NKV, D), dtype=np.float32)
        return torch.from_numpy(r).to(torch.bfloat16)

    def extend(self, sid, new_tokens):
        """Append tokens; returns the K/V rows [n, NKV, D] of the new positions."""
        h = self.h.get(sid, 0x5EED)
        ks, vs = [], []
        for t in new_tokens:
            h = zlib.crc32(np.int64(t).tobytes(), h)  # rolling hash of the prefix
            kv = self._rows(h)
            ks.append(kv[0])
            vs.append(kv[1])
        self.h[sid] = h
        self.toks.setdefault(sid, []).extend(new_tokens)
        self.k.setdefault(sid, []).extend(ks)
        self.v.setdefault(sid, []).extend(vs)
        if not ks:
            return None, None
        return torch.stack(ks), torch.stack(vs)


def oracle_attention(model, ids, q, fp8, k_scale, v_scale):
    """fp64 attention over each sequence's logical K/V in private blocks."""
    lens = [len(model.toks[s]) for s in ids]
    nblk = sum(-(-n // BS) for n in lens)
    maxb = max(-(-n // BS) for n in lens)
    fill = 0x7F if fp8 else 0x7FC0
    kp = O.new_pool(nblk, NKV, BS, D, fp8, fill)
    vp = O.new_pool(nblk, NKV, BS, D, fp8, fill)
    tables = np.full((len(ids), maxb), -1, np.int32)
    base = 0
    for r, s in enumerate(ids):
        nb = -(-lens[r] // BS)
        tables[r, :nb] = np.arange(base, base + nb)
        slots = torch.arange(base * BS, base * BS + lens[r], dtype=torch.int32)
        st = O.store_kvcache(torch.stack(model.k[s]), torch.stack(model.v[s]), kp, vp, slots, nblk, BS,
                             k_scale, v_scale)
        assert st == O.ORC_OK
        base += nb
    out, st = O.paged_attention_decode(q.cpu(), kp, vp, tables, np.array(lens, np.int32), NKV, BS,
                                       1.0 / math.sqrt(D), k_scale, v_scale, num_threads=8)
    assert st == O.ORC_OK
    return out


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
def test_manager_drives_store_and_decode(fp8):
    dev = "cuda"
    rng = np.random.default_rng(11)
    num_blocks = 768
    bm = BlockManager(num_blocks, BS)
    model = Model()
    shape = (num_blocks, NKV, BS, D)
    if fp8:
        kp = torch.full(shape, 0x7F, dtype=torch.uint8, device=dev)
        vp = torch.full(shape, 0x7F, dtype=torch.uint8, device=dev)
        k_scale = torch.full((NKV,), 0.02, dtype=torch.float32)
        v_scale = torch.full((NKV,), 0.03, dtype=torch.float32)
        ksd, vsd = k_scale.to(dev), v_scale.to(dev)
    else:
        kp = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        vp = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        k_scale = v_scale = ksd = vsd = None
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def admit(sid, toks):
        st, cached = bm.add_sequence(sid, toks)
        assert st == K.PKV_OK
        k, v = model.extend(sid, toks)
        slots = torch.tensor(bm.slots(sid, cached, len(toks) - cached), dtype=torch.int32, device=dev)
        if slots.numel():  # only the uncached tokens are written
            K.store_kvcache(k[cached:].to(dev), v[cached:].to(dev), kp, vp, slots, ksd, vsd, err)
        return cached

    prompts = [rng.integers(0, 32000, n).tolist() for n in (700, 420, 333, 1000)]
    live, next_id, hit_tokens = [], 0, 0
    for i in range(24):
        p = prompts[i % 4]
        toks = p[: len(p) - int(rng.integers(0, 200))] + rng.integers(0, 32000, int(rng.integers(1, 40))).tolist()
        hit_tokens += admit(next_id, toks)
        live.append(next_id)
        next_id += 1
    assert hit_tokens > 0

    scale = 1.0 / math.sqrt(D)
    for step in range(40):
        if step == 20:  # some requests end; new ones reuse their (still cached) prefixes
            for sid in live[::3]:
                assert bm.free_sequence(sid) == K.PKV_OK
            live = [s for s in live if s not in live[::3]]
            for i in range(6):
                toks = prompts[i % 4][:512] + [int(rng.integers(0, 32000))]
                assert admit(next_id, toks) >= 256
                live.append(next_id)
                next_id += 1
        new = rng.integers(0, 32000, len(live)).tolist()
        slots = bm.append_tokens(live, new)
        ks, vs = zip(*(model.extend(s, [t]) for s, t in zip(live, new)))
        K.store_kvcache(torch.cat(ks).to(dev), torch.cat(vs).to(dev), kp, vp, torch.from_numpy(slots).to(dev),
                        ksd, vsd, err)
        maxb = max(-(-len(model.toks[s]) // BS) for s in live)
        tables, lens = bm.block_tables(live, maxb)
        q = torch.from_numpy(rng.standard_normal((len(live), NQ, D), dtype=np.float32)).to(torch.bfloat16)
        out = K.paged_attention_decode(q.to(dev), kp, vp, torch.from_numpy(tables).to(dev),
                                       torch.from_numpy(lens).to(dev), scale, k_scale=ksd, v_scale=vsd,
                                       max_context_len=int(lens.max()), dev_err=err)
        if step in (0, 19, 39):
            assert K.read_device_error(err) == K.PKV_OK
            ref = oracle_attention(model, live, q, fp8, k_scale, v_scale)
            compare(out, ref, fp8, f"step {step}")
    assert bm.num_free() + len({b for s in live for b in bm.block_table(s)[0]}) == num_blocks
    assert BF16_ABS > 0
