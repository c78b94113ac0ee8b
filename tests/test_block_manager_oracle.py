"""The reference block manager against its pins, and planted mistakes in copies
of it that the pins must catch (no GPU)."""

import importlib.util
import os
import sys
import tempfile

import pytest

import block_manager_pins as P
from oracle.block_manager import BlockManagerOracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "block_manager.py")


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(BlockManagerOracle)


# (name, original text, mutated text)
MUTANTS = [
    ("matching goes on after a miss", "            if b is None:\n                break", "            if b is None:\n                continue"),
    ("hit does not take a reference", "            self.ref[b] += 1\n        table", "            pass\n        table"),
    ("shared block freed too early", "            if self.ref[b] == 0:\n                self.free.append(b)", "            if True:\n                self.free.append(b)"),
    ("reused block keeps its cache entry", "        if b in self.key_of:  # its cached content is about to be overwritten\n            del self.cached[self.key_of.pop(b)]", "        pass"),
    ("partial blocks shared", [
        ("            if len(self.content[b]) == bs:\n                self._register(b, tuple(tokens[: (i + 1) * bs]))", "            self._register(b, tuple(tokens[: (i + 1) * bs]))"),
        ("        for i in range(len(tokens) // bs):", "        for i in range(n_blocks):"),
    ], None),
    ("key without the prefix", "            b = self.cached.get(tuple(tokens[: (i + 1) * bs]))", "            b = self.cached.get(tuple(tokens[i * bs : (i + 1) * bs]))"),
    ("free queue LIFO", "        b = self.free.pop(0)", "        b = self.free.pop()"),
    ("first block freed first", "        for b in reversed(s[\"table\"]):", "        for b in s[\"table\"]:"),
    ("hit length in blocks", "        return OK, len(hits) * bs", "        return OK, len(hits)"),
    ("slot offset", "        return OK, b * bs + n % bs", "        return OK, b * bs + n // bs"),
    ("new block one token late", "        if n % bs == 0:\n            if not self.free:", "        if n % bs == 1:\n            if not self.free:"),
    ("filled block not cached", "        if len(self.content[b]) == bs:\n            self._register(b, tuple(s[\"tokens\"]))", "        pass"),
    ("failure half-applies", "        if len(self.free) - free_hits < n_blocks - len(hits):\n            return ERR_NO_BLOCKS, 0", "        if len(self.free) - free_hits < 0:\n            return ERR_NO_BLOCKS, 0"),
]


def _load_mutant(src):
    d = tempfile.mkdtemp()
    path = os.path.join(d, "bm_mutant.py")
    with open(path, "w") as f:
        f.write(src)
    spec = importlib.util.spec_from_file_location("bm_mutant_%d" % abs(hash(src)), path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.BlockManagerOracle


def _edits(old, new):
    return old if new is None else [(old, new)]


def test_mutation_sites_exist():
    src = open(SRC).read()
    for name, old, new in MUTANTS:
        for o, _ in _edits(old, new):
            assert src.count(o) == 1, name


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    src = open(SRC).read()
    for o, n in _edits(old, new):
        src = src.replace(o, n)
    cls = _load_mutant(src)
    assert P.run_all(cls), f"no pin catches: {name}"
