"""Planted mistakes, on the CPU, in copies of the oracle: each mutant takes the source of
``oracle/attention.py``, changes one thing that a plausible slip would change (a dropped
scale or term, a wrong sign, index, offset or exponent bias, a transposed or swapped
operand, a missing guard or clamp), and must fail at least one pin of ``test_oracle.py``;
the unchanged copy must pass every pin.  The oracle's file is never modified: the copy is
compiled into a fresh namespace, its functions stand in for the package's exports while a
fresh copy of the pin module runs, and the package is restored afterwards."""
import ast
import importlib.util
import inspect
import itertools
import os
import sys
import types

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
# the module itself (the package re-exports a function of the same name as its attribute)
SRC = inspect.getsource(sys.modules["oracle.attention"])

# (what, function the text must sit in, text in the oracle's source, replacement); the first
# occurrence of the text is replaced
MUTANTS = [
    ("dropped scale", "_softmax_attend", "s = scale * (qm @ km.T)", "s = (qm @ km.T)"),
    ("V in place of K in the scores", "_softmax_attend", "s = scale * (qm @ km.T)", "s = scale * (qm @ vm.T)"),
    ("causal offset off by one", "_visible", "j[None, :] <= (rows[:, None] + (Sk - Sq))",
     "j[None, :] < (rows[:, None] + (Sk - Sq))"),
    ("top-left causal alignment", "_visible", "j[None, :] <= (rows[:, None] + (Sk - Sq))",
     "j[None, :] <= rows[:, None]"),
    ("LSE without the max", "_softmax_attend", "lse[has] = m + np.log(z)", "lse[has] = np.log(z)"),
    ("LSE in log2", "_softmax_attend", "lse[has] = m + np.log(z)", "lse[has] = m + np.log2(z)"),
    ("unnormalised output", "_softmax_attend", "o[has] = (e @ vm) / z[:, None]", "o[has] = (e @ vm)"),
    ("wrong sign in the exponent", "_softmax_attend", "e = np.exp(sh - m[:, None])", "e = np.exp(m[:, None] - sh)"),
    ("interleaved GQA mapping", "attention", "kvh = h // G", "kvh = h % Hkv"),
    ("no guard for rows without a key", "_softmax_attend", "has = vis.any(axis=1)", "has = np.ones(n, dtype=bool)"),
    ("merge weights without the reference", "combine_lse", "w = np.exp(lses - ref)", "w = np.exp(lses)"),
    ("merge LSE without the reference", "combine_lse", "ref + np.log(np.where(den > 0, den, 1.0))",
     "np.log(np.where(den > 0, den, 1.0))"),
    ("paged decode: page and row swapped", "decode_paged", "kb = _f64(k_cache)[pages, t % page_size]",
     "kb = _f64(k_cache)[pages, t // page_size % page_size]"),
    ("paged decode: lengths not clamped", "decode_paged",
     "n = int(min(max(int(seqlens[b]), 0), page_size * bt.shape[1]))", "n = int(max(int(seqlens[b]), 0))"),
    ("varlen: last key of each sequence dropped", "attention_varlen",
     "o, lse = attention(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], scale, causal)",
     "o, lse = attention(q[None, q0:q1], k[None, k0:k1 - 1], v[None, k0:k1 - 1], scale, causal)"),
    ("varlen: keys taken at the query offsets", "attention_varlen",
     "o, lse = attention(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], scale, causal)",
     "o, lse = attention(q[None, q0:q1], k[None, q0:q0 + k1 - k0], v[None, q0:q0 + k1 - k0], scale, causal)"),
    ("block-sparse: mask transposed (square masks)", "attention_block_sparse",
     "vis = base & bm[b, h][rows[:, None], cols[None, :]]",
     "vis = base & (bm[b, h].T if nq == nk else bm[b, h])[rows[:, None], cols[None, :]]"),
    ("block-sparse: mask ignored", "attention_block_sparse",
     "vis = base & bm[b, h][rows[:, None], cols[None, :]]", "vis = base"),
    ("backward: Delta dropped", "attention_backward", "ds = p * (dp - delta[:, None])", "ds = p * dp"),
    ("backward: dQ without the scale", "attention_backward", "dq[b, :, h, :] = scale * (ds @ km)",
     "dq[b, :, h, :] = ds @ km"),
    ("backward: dV from the scores' transpose", "attention_backward", "dv[b, :, kvh, :] += p.T @ dom",
     "dv[b, :, kvh, :] += (p.T @ dom) * 0.5 + (p.T @ dom)[::-1] * 0.5"),
    ("e4m3: exponent bias 8", "decode_e4m3", "np.exp2(e.astype(np.float64) - 7.0)", "np.exp2(e.astype(np.float64) - 8.0)"),
    ("e4m3: subnormal step 2^-10", "decode_e4m3", "m * 2.0 ** -9", "m * 2.0 ** -10"),
    ("FP8: descale divides", "attention_fp8", "return attention(decode_e4m3(q8) * q_descale",
     "return attention(decode_e4m3(q8) / q_descale"),
    ("FP8: V descale on K", "attention_fp8", "decode_e4m3(k8) * k_descale, decode_e4m3(v8) * v_descale,\n",
     "decode_e4m3(k8) * v_descale, decode_e4m3(v8) * v_descale,\n"),
    ("paged prefill: lengths not clamped", "attention_paged_prefill",
     "n = int(min(max(int(seqlens_k[b]), 0), page_size * bt.shape[1]))", "n = int(max(int(seqlens_k[b]), 0))"),
    ("blockwise: accumulator not rescaled", "attention_blockwise", "acc = acc * alpha[:, None] + p @ v",
     "acc = acc + p @ v"),
    ("blockwise: denominator not rescaled", "attention_blockwise", "l = l * alpha + p.sum(axis=1)",
     "l = l + p.sum(axis=1)"),
]
# (Not listed: the recurrence without its -inf guard.  The guard only matters for a row whose
# keys are all masked, and those rows are zeroed by the final l > 0 test either way, so that
# change computes the same results: no pin can or needs to tell it apart.)


def body_of(src, func):
    """The function's syntax tree without its docstring, as text."""
    node = next(n for n in ast.parse(src).body if isinstance(n, ast.FunctionDef) and n.name == func)
    body = node.body[1:] if (node.body and isinstance(node.body[0], ast.Expr)
                             and isinstance(node.body[0].value, ast.Constant)) else node.body
    return ast.dump(ast.Module(body=body, type_ignores=[]))


def build(func=None, old=None, new=None):
    src = SRC
    if old is not None:
        at = src.find(old)
        assert at >= 0, old
        start = src.rfind("\ndef ", 0, at)
        assert src[start + 5:].startswith(func + "("), (old, func)
        src = src[:at] + new + src[at + len(old):]
        assert body_of(src, func) != body_of(SRC, func), "the change must reach the code, not only its text"
    mod = types.ModuleType("oracle_copy")
    exec(compile(src, "<oracle copy>", "exec"), mod.__dict__)
    return mod


def pin_calls(pins):
    """Every test function of the pin module with each of its parameter sets."""
    out = []
    for name, fn in vars(pins).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        grids = []
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            names = [n.strip() for n in mark.args[0].split(",")] if isinstance(mark.args[0], str) else list(mark.args[0])
            vals = [v if len(names) > 1 else (v,) for v in mark.args[1]]
            grids.append([dict(zip(names, v)) for v in vals])
        for combo in itertools.product(*grids) if grids else [()]:
            kw = {}
            for d in combo:
                kw.update(d)
            out.append((name, fn, kw))
    return out


def failed_pins(mod, monkeypatch, stop_at_first):
    for name in oracle.__all__:
        monkeypatch.setattr(oracle, name, getattr(mod, name))
    spec = importlib.util.spec_from_file_location("oracle_pins_copy", os.path.join(HERE, "test_oracle.py"))
    pins = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(pins)            # its `from oracle import ...` now binds the copy
    failed = []
    for name, fn, kw in pin_calls(pins):
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except pytest.skip.Exception:
            continue
        except Exception:        # a mismatch, a NaN, an error: the pin rejects the copy
            failed.append(name)
            if stop_at_first:
                break
    return failed


def test_unchanged_copy_passes_every_pin(monkeypatch):
    assert failed_pins(build(), monkeypatch, stop_at_first=False) == []


@pytest.mark.parametrize("what,func,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(what, func, old, new, monkeypatch):
    assert failed_pins(build(func, old, new), monkeypatch, stop_at_first=True), f"no pin catches: {what}"
