"""Plant plausible mistakes in copies of the oracle; each must fail a pin.

Every mutant below is a one-line change to ``oracle/pkv_oracle.c`` of the
kind a reader could miss: a dropped term, a wrong index or sign, swapped
operands, a transposed layout, a wrong rounding tie. The copy is compiled and
the whole pin suite runs against it in a child process (so a crash counts as
caught). If a mutant survived, the pins would not be pinning that line.
"""

import json
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "pkv_oracle.c")

# (name, original text, mutated text, which occurrence (0-based) to change)
MUTANTS = [
    ("rope sin sign", "ya = fmaf(-xb, s, xa * c);", "ya = fmaf(xb, s, xa * c);", 0),
    ("rope partner", "*b = i + head_dim / 2;", "*b = head_dim - 1 - i;", 0),
    ("rope cos for sin", "s = cos_sin[m * head_dim + head_dim / 2 + i];", "s = cos_sin[m * head_dim + i];", 0),
    ("rope angle index", "c = cos_sin[m * head_dim + i];", "c = cos_sin[m * head_dim + head_dim / 2 - 1 - i];", 0),
    ("rope position off by one", "int64_t m = positions[t];", "int64_t m = positions[t] > 0 ? positions[t] - 1 : 0;",
     0),
    ("rope pairings swapped", "if (style == 1) {", "if (style == 0) {", 0),
    ("rope store unrotated k", "st = orc_store_kvcache(k_rot, v,", "st = orc_store_kvcache(k, v,", 0),
    ("rope bad position stored", "slots[t] = bad ? -1 : slot_mapping[t];", "slots[t] = slot_mapping[t];", 0),
    ("gqa interleaved", "int g = h / group;", "int g = h % num_kv_heads;", 0),
    ("offset from division", "int off = t % block_size;", "int off = (t / block_size) % block_size;", 0),
    ("block from offset", "int64_t blk = table[t / block_size];", "int64_t blk = table[t % block_size];", 0),
    ("pv offset", "int off = t % block_size;", "int off = (t + 1) % block_size;", 1),
    ("scale dropped", "score[t] = (double)scale * dot;", "score[t] = dot;", 0),
    ("max not subtracted", "w[t] = exp(score[t] - m);", "w[t] = exp(score[t]);", 0),
    ("not normalised", "acc[i] / z;", "acc[i];", 0),
    ("last token dropped", "for (t = 0; t < ctx; ++t) {\n                w[t]",
     "for (t = 0; t < ctx - 1; ++t) {\n                w[t]", 0),
    ("v read from k", "cache_value(v_cache, idx, fp8, v_scale, g,", "cache_value(k_cache, idx, fp8, v_scale, g,", 0),
    ("q head of kv head", "q + ((int64_t)s * num_q_heads + h) * head_dim", "q + ((int64_t)s * num_q_heads + g) * head_dim", 0),
    ("layout transposed", "((blk * nkv + h) * bs + off)", "((blk * bs + off) * nkv + h)", 0),
    ("slot zero skipped", "if (slot < 0)", "if (slot <= 0)", 0),
    ("k and v swapped", "((uint16_t *)k_cache)[dst] = k[src];", "((uint16_t *)k_cache)[dst] = v[src];", 0),
    ("fp8 scale unused on read", "* (double)scale[h];", ";", 0),
    ("fp8 scale multiplies on store", "float ky = kx / ks;", "float ky = kx * ks;", 0),
    ("fp8 ties away", "(d_hi == d_lo && (lo & 1))", "(d_hi == d_lo)", 0),
    ("fp8 saturation drops sign", "return sign | 0x7E;", "return 0x7E;", 0),
    ("fp8 subnormal exponent", "ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)", 0),
    ("fp8 bias", "e - 7);", "e - 8);", 0),
    ("bf16 widening", "(uint32_t)bits << 16;", "(uint32_t)bits << 15;", 0),
    ("bounds check off by one", "ctx > max_blocks_per_seq * block_size", "ctx > max_blocks_per_seq * block_size + 1", 0),
    ("block id check", "table[t / block_size] >= num_blocks", "table[t / block_size] > num_blocks", 0),
    # chunked prefill
    ("prefill gqa interleaved", "int g = h / group;", "int g = h % num_kv_heads;", 1),
    ("prefill sees one future token", "int p = ctx - c + r;", "int p = ctx - c + r + 1;", 0),
    ("prefill ignores the history", "int p = ctx - c + r;", "int p = r;", 0),
    ("prefill mask excludes itself", "for (t = 0; t <= p; ++t) {\n                    w[t]",
     "for (t = 0; t < p; ++t) {\n                    w[t]", 0),
    ("prefill q row without offset", "q + (row * num_q_heads + h) * head_dim", "q + ((int64_t)r * num_q_heads + h) * head_dim", 0),
    ("prefill out row without offset", "out + (row * num_q_heads + h) * head_dim", "out + ((int64_t)r * num_q_heads + h) * head_dim", 0),
    ("prefill chunk longer than context", "bad = (ctx < c || ctx > max_blocks_per_seq * block_size);",
     "bad = (ctx > max_blocks_per_seq * block_size);", 0),
    ("prefill decreasing offsets accepted", "if (cu_q_lens[s + 1] < cu_q_lens[s])", "if (0)", 0),
    ("prefill max not subtracted", "w[t] = exp(score[t] - m);", "w[t] = exp(score[t]);", 1),
    ("prefill not normalised", "acc[i] / z;", "acc[i];", 1),
    ("prefill v read from k", "cache_value(v_cache, idx, fp8, v_scale, g,", "cache_value(k_cache, idx, fp8, v_scale, g,", 1),
    # E4M3 with per-token scales
    ("token scale read per head", "        return orc_e4m3_to_double(((const uint8_t *)cache)[idx]) * (double)scale[sidx];",
     "        return orc_e4m3_to_double(((const uint8_t *)cache)[idx]) * (double)scale[h];", 0),
    ("token scale amax without abs", "ka = fmaxf(ka, fabsf((float)orc_bf16_to_double(k[src])));",
     "ka = fmaxf(ka, (float)orc_bf16_to_double(k[src]));", 0),
    ("token scale 240", "ks = ka / 448.0f;", "ks = ka / 240.0f;", 0),
    ("token scale no floor", "if (ks < FLT_MIN)\n                    ks = FLT_MIN;", "if (0)\n                    ks = FLT_MIN;", 0),
    ("token scale wrong slot", "return (blk * nkv + h) * bs + off;", "return (blk * nkv + h) * bs + (off + 1) % bs;", 0),
    ("token scale v from k", "vs = va / 448.0f;", "vs = ka / 448.0f;", 0),
    # add + RMSNorm
    ("rmsnorm eps outside sqrt", "inv = 1.0 / sqrt(ss / hidden + eps);", "inv = 1.0 / (sqrt(ss / hidden) + eps);", 0),
    ("rmsnorm sum not mean", "inv = 1.0 / sqrt(ss / hidden + eps);", "inv = 1.0 / sqrt(ss + eps);", 0),
    ("rmsnorm n - 1", "inv = 1.0 / sqrt(ss / hidden + eps);", "inv = 1.0 / sqrt(ss / (hidden - 1) + eps);", 0),
    ("rmsnorm residual not added", "h += orc_bf16_to_double(residual[row + i]);", "h += 0.0;", 0),
    ("rmsnorm residual out is x", "residual_out[row + i] = orc_bf16_from_double(out[row + i]);",
     "residual_out[row + i] = x[row + i];", 0),
    ("rmsnorm weight unused", "out[row + i] = orc_bf16_to_double(weight[i]) * (out[row + i] * inv);",
     "out[row + i] = out[row + i] * inv;", 0),
    ("rmsnorm abs not square", "ss += h * h;", "ss += fabs(h);", 0),
    ("bf16 rounding ties away", "(r == 0.5 && fmod(fl, 2.0) == 1.0)", "(r == 0.5)", 0),
    ("bf16 subnormal spacing", "quantum = ldexp(1.0, -133);", "quantum = ldexp(1.0, -132);", 0),
    ("bf16 overflow kept finite", "return sign | 0x7F80;", "return sign | 0x7F7F;", 0),
    ("bf16 sign of zero", "uint16_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x8000 : 0;",
     "uint16_t sign = (v < 0) ? 0x8000 : 0;", 0),
]


def _mutate(src: str, old: str, new: str, which: int) -> str:
    pos = -1
    for _ in range(which + 1):
        pos = src.find(old, pos + 1)
        assert pos >= 0, f"mutation site not found: {old!r}"
    return src[:pos] + new + src[pos + len(old):]


def _run_mutant(args):
    name, old, new, which, tmp = args
    src = open(SRC).read()
    path = os.path.join(tmp, name.replace(" ", "_") + ".c")
    with open(path, "w") as f:
        f.write(_mutate(src, old, new, which))
    lib = path[:-2] + ".so"
    O.build(path, lib, force=True)
    r = subprocess.run([sys.executable, os.path.join(HERE, "_oracle_pin_runner.py"), lib],
                       capture_output=True, text=True, timeout=600)
    if r.returncode != 0:
        return name, [f"crashed (rc={r.returncode})"]
    return name, json.loads(r.stdout.strip().splitlines()[-1])


def test_mutation_sites_exist():
    src = open(SRC).read()
    for name, old, _, which in MUTANTS:
        assert src.count(old) > which, name


def test_unmutated_copy_passes_every_pin(tmp_path):
    lib = str(tmp_path / "clean.so")
    O.build(SRC, lib, force=True)
    r = subprocess.run([sys.executable, os.path.join(HERE, "_oracle_pin_runner.py"), lib],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert json.loads(r.stdout.strip().splitlines()[-1]) == []


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(_run_mutant, [(*m, tmp) for m in MUTANTS]))
    survivors = [name for name, failed in results if not failed]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
