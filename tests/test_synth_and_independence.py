"""The seeded input generators, and the separation between the oracle and the CUDA path.

synth.py is the one module both sides use: it must be deterministic per seed, draw what its
docstrings state, and hold no attention arithmetic.  The oracle and the product path share
nothing else: neither imports the other, no C/CUDA source of one includes a file of the
other, and bench.py touches the oracle only in its CPU-baseline / reference timing.
"""
import ast
import math
import os
import re

import numpy as np
import torch

from long_context_04_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# ----------------------------------------------------------------------------- synth
def test_draws_are_deterministic_per_seed():
    a = synth.qkv(64, 2, 64, seed=3, dtype=torch.float32)
    b = synth.qkv(64, 2, 64, seed=3, dtype=torch.float32)
    c = synth.qkv(64, 2, 64, seed=4, dtype=torch.float32)
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y)
        assert not torch.equal(x, z)
    q, k, v = a
    assert not torch.equal(q, k) and not torch.equal(k, v)      # three separate draws


def test_qkv_distribution():
    D = 128
    q, _, _ = synth.qkv(4096, 4, D, seed=0, dtype=torch.float32)
    x = q.double()
    assert abs(float(x.mean())) < 3e-3
    assert abs(float(x.std()) - 1 / math.sqrt(D)) < 2e-3
    qb, _, _ = synth.qkv(4096, 4, D, seed=0, dtype=torch.bfloat16)
    assert qb.dtype == torch.bfloat16
    assert torch.equal(qb, q.to(torch.bfloat16))                 # drawn in fp32, then cast


def test_cu_seqlens_uniform():
    for total, S, seed in [(1000, 7, 0), (262144, 8, 0), (5, 12, 1), (0, 3, 2)]:
        cu = synth.cu_seqlens_uniform(total, S, seed=seed)
        assert cu.dtype == np.int32 and len(cu) == S + 1
        assert cu[0] == 0 and cu[-1] == total and bool(np.all(np.diff(cu) >= 0))
        assert np.array_equal(cu, synth.cu_seqlens_uniform(total, S, seed=seed))


def test_decode_tokens_and_initial_state():
    a = synth.decode_tokens(4, 2, 64, step=0, seed=0, dtype=torch.float32)
    b = synth.decode_tokens(4, 2, 64, step=1, seed=0, dtype=torch.float32)
    c = synth.decode_tokens(4, 2, 64, step=0, seed=1, dtype=torch.float32)
    assert all(x.shape == (4, 2, 64) for x in a)
    assert not torch.equal(a[0], b[0]) and not torch.equal(a[0], c[0])
    assert torch.equal(a[0], synth.decode_tokens(4, 2, 64, step=0, seed=0, dtype=torch.float32)[0])
    D, tokens = 64, 400
    x = synth.initial_state(3, 2, D, tokens=tokens, seed=5)
    assert x.shape == (3, 2, D, D) and x.dtype == torch.float32
    assert abs(float(x.double().std()) - math.sqrt(tokens) / D) < 0.02 * math.sqrt(tokens) / D
    assert torch.equal(x, synth.initial_state(3, 2, D, tokens=tokens, seed=5))


def test_synth_holds_no_attention_arithmetic():
    tree = ast.parse(open(os.path.join(ROOT, "long_context_04_b200", "synth.py")).read())
    imported = {a.name.split(".")[0] for n in ast.walk(tree) if isinstance(n, ast.Import) for a in n.names}
    imported |= {n.module.split(".")[0] for n in ast.walk(tree) if isinstance(n, ast.ImportFrom) and n.module}
    assert imported <= {"__future__", "math", "numpy", "torch"}, imported
    src = open(os.path.join(ROOT, "long_context_04_b200", "synth.py")).read()
    for word in ("matmul", "einsum", "cumsum", "bmm", " @ ", "oracle"):
        assert word not in src, word


# ----------------------------------------------------------------------------- independence
def _py_imports(path):
    tree = ast.parse(open(path).read())
    out = []
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out += [(a.name, node) for a in node.names]
        elif isinstance(node, ast.ImportFrom):
            out.append((("." * node.level) + (node.module or ""), node))
    return out


def _files(sub, exts):
    d = os.path.join(ROOT, sub)
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith(exts)]


def test_oracle_imports_nothing_of_the_product():
    for path in _files("oracle", (".py",)):
        for name, _ in _py_imports(path):
            assert not name.startswith("long_context_04_b200"), (path, name)


def test_product_imports_nothing_of_the_oracle():
    for path in _files("long_context_04_b200", (".py",)):
        for name, _ in _py_imports(path):
            assert name.split(".")[0] != "oracle", (path, name)


def test_native_sources_include_nothing_of_each_other():
    inc = re.compile(r'#\s*include\s*"([^"]+)"')
    for path in _files("oracle", (".c", ".h")):
        for target in inc.findall(open(path).read()):
            assert "csrc" not in target and "include/" not in target and "lightning" not in target, (path, target)
    for path in _files(os.path.join("long_context_04_b200", "csrc"), (".cu", ".cuh")):
        for target in inc.findall(open(path).read()):
            assert "oracle" not in target, (path, target)


def test_bench_uses_the_oracle_only_for_the_cpu_timing():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    # the only functions that may use the oracle: the CPU-baseline timings
    allowed = {"time_oracle_prefill", "cpu_oracle_prefill", "cpu_oracle_quadratic", "decode_cpu_baseline"}
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                names = []
                if isinstance(node, ast.Import):
                    names = [a.name for a in node.names]
                elif isinstance(node, ast.ImportFrom):
                    names = [node.module or ""]
                if any(n.split(".")[0] == "oracle" for n in names):
                    assert fn.name in allowed, fn.name
    # and no module-level import of it
    for node in tree.body:
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
            assert all(n.split(".")[0] != "oracle" for n in names)
    # time_oracle_prefill is reached only from the CPU-baseline and reference legs
    callers = {fn.name for fn in ast.walk(tree) if isinstance(fn, ast.FunctionDef)
               for node in ast.walk(fn) if isinstance(node, ast.Call)
               and getattr(node.func, "id", None) == "time_oracle_prefill"}
    assert callers == {"cpu_baseline", "run_reference"}, callers

    def callers_of(name):
        return {fn.name for fn in ast.walk(tree) if isinstance(fn, ast.FunctionDef)
                for node in ast.walk(fn) if isinstance(node, ast.Call)
                and getattr(node.func, "id", None) == name}
    # the per-config baselines run inside bench_configs only under its `cpu` switch, and the
    # decode baseline only on rank 0 of a 1-GPU run
    assert callers_of("cpu_oracle_prefill") == {"bench_configs"}
    assert callers_of("cpu_oracle_quadratic") == {"bench_configs"}
    assert callers_of("decode_cpu_baseline") == {"run_ours"}
    cfg = next(fn for fn in ast.walk(tree) if isinstance(fn, ast.FunctionDef) and fn.name == "bench_configs")
    for node in ast.walk(cfg):
        if isinstance(node, ast.Call) and getattr(node.func, "id", "") in ("cpu_oracle_prefill", "cpu_oracle_quadratic"):
            guarded = any(isinstance(i, ast.If) and isinstance(i.test, ast.Name) and i.test.id == "cpu"
                          and any(c is node for c in ast.walk(i)) for i in ast.walk(cfg))
            assert guarded, "a per-config CPU baseline outside the `if cpu:` switch"
