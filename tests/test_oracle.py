"""CPU tests of the FP64 oracle against its pins (no GPU needed)."""
from __future__ import annotations

import math
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from oracle_pins import ALL_PINS, failing_pins
from scaled_dot_product_10_b200.workloads import make_qkv


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(lib, pin):
    pin(lib)


def _brute_force(q, k, v, causal, scale, window_left=-1):
    """Per-element scalar evaluation in pure Python floats (tiny shapes only)."""
    qq = q.float().double().tolist()
    kk = k.float().double().tolist()
    vv = v.float().double().tolist()
    b, s_q, h_q, d = q.shape
    _, s_k, h_kv, _ = k.shape
    grp = h_q // h_kv
    o = np.zeros((b, h_q, s_q, d))
    lse = np.zeros((b, h_q, s_q))
    for bi in range(b):
        for h in range(h_q):
            g = h // grp
            for i in range(s_q):
                scores = []
                for j in range(s_k):
                    if causal and j > i + (s_k - s_q):  # bottom-right aligned
                        continue
                    if window_left >= 0 and j < i + (s_k - s_q) - window_left:
                        continue
                    acc = 0.0
                    for c in range(d):
                        acc += qq[bi][i][h][c] * kk[bi][j][g][c]
                    scores.append((j, acc * scale))
                mx = max(sv for _, sv in scores)
                w = [(j, math.exp(sv - mx)) for j, sv in scores]
                tot = sum(x for _, x in w)
                for c in range(d):
                    o[bi, h, i, c] = sum(x * vv[bi][j][g][c] for j, x in w) / tot
                lse[bi, h, i] = mx + math.log(tot)
    return o, lse


@pytest.mark.parametrize("shape", [(1, 1, 1, 5, 5, 4), (2, 4, 2, 17, 17, 4), (1, 2, 1, 9, 9, 128),
                                   (1, 2, 2, 4, 11, 4), (2, 2, 1, 1, 6, 8)])
def test_oracle_brute_force(lib, shape):
    b, h_q, h_kv, s_q, s_k, d = shape
    q, k, v = make_qkv(b, h_q, h_kv, s_q, s_k, seed=31 + s_q + s_k, d=d)
    for causal in (False, True):
        o, lse, _ = oracle.attn_fwd(q, k, v, causal, 0.3, lib=lib)
        ob, lb = _brute_force(q, k, v, causal, 0.3)
        assert np.max(np.abs(o - ob)) < 1e-12
        assert np.max(np.abs(lse - lb)) < 1e-12


@pytest.mark.parametrize("shape,window", [((1, 2, 1, 7, 7, 4), 2), ((2, 2, 2, 5, 12, 8), 3),
                                          ((1, 1, 1, 9, 9, 4), 0)])
def test_oracle_brute_force_window(lib, shape, window):
    b, h_q, h_kv, s_q, s_k, d = shape
    q, k, v = make_qkv(b, h_q, h_kv, s_q, s_k, seed=51 + s_q + window, d=d)
    o, lse, _ = oracle.attn_fwd(q, k, v, True, 0.3, lib=lib, window_left=window)
    ob, lb = _brute_force(q, k, v, True, 0.3, window_left=window)
    assert np.max(np.abs(o - ob)) < 1e-12
    assert np.max(np.abs(lse - lb)) < 1e-12


def test_oracle_rejects_bad_arguments(lib):
    q, k, v = make_qkv(1, 4, 3, 8, 8, seed=1, d=4)   # 4 % 3 != 0
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, False, 1.0, lib=lib)
    q, k, v = make_qkv(1, 2, 2, 8, 4, seed=1, d=4)   # causal with s_q > s_k
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, True, 1.0, lib=lib)


# Planted mistakes: each is a plausible slip in the oracle's arithmetic.  A
# mutant oracle is built from a copy of the source in a temporary directory
# and must fail at least one pin.
MUTANTS = {
    "dropped_scale": ("Srow[j] = scale * dot;", "Srow[j] = dot;"),
    "mask_wrong_side": ("if (causal && j > i + off)", "if (causal && j < i + off)"),
    "mask_off_by_one": ("if (causal && j > i + off)", "if (causal && j > i + off + 1)"),
    "mask_top_left": ("if (causal && j > i + off)", "if (causal && j > i)"),
    "mask_offset_sign": ("const int off = s_k - s_q;", "const int off = s_q - s_k;"),
    "gqa_modulo_mapping": ("const int g = h / group;", "const int g = h % h_kv;"),
    "transposed_scores": ("dot += Qb[(int64_t)i * q_row_stride + c] *\n                       Kb[(int64_t)j * kv_row_stride + c];",
                          "dot += Qb[(int64_t)j * q_row_stride + c] *\n                       Kb[(int64_t)i * kv_row_stride + c];"),
    "dropped_first_term": ("for (int c = 0; c < d; ++c)\n                dot +=", "for (int c = 1; c < d; ++c)\n                dot +="),
    "no_max_subtraction": ("Srow[j] = exp(Srow[j] - m);", "Srow[j] = exp(Srow[j]);"),
    "exp_sign_flip": ("Srow[j] = exp(Srow[j] - m);", "Srow[j] = exp(m - Srow[j]);"),
    "min_instead_of_max": ("if (Srow[j] > m) m = Srow[j];", "if (Srow[j] < m) m = Srow[j];"),
    "no_normalisation": ("Srow[j] = Srow[j] / l;", "Srow[j] = Srow[j];"),
    "lse_missing_max": ("m + log(l);", "log(l);"),
    "lse_log2": ("m + log(l);", "m + log2(l);"),
    "k_used_as_v": ("const double *vrow = Vb +", "const double *vrow = Kb +"),
    "mask_to_zero": ("Srow[j] = -INFINITY;", "Srow[j] = 0.0;"),
    "window_off_by_one": ("j < i + off - window_left)", "j < i + off - window_left + 1)"),
    "window_wrong_side": ("j < i + off - window_left)", "j > i + off - window_left)"),
    "bf16_decode_shift": ("((uint32_t)bits) << 16", "((uint32_t)bits) << 15"),
    # backward
    "bwd_dq_dropped_scale": ("dQb[(int64_t)i * qs + c] = scale * acc;",
                             "dQb[(int64_t)i * qs + c] = acc;"),
    "bwd_dk_dropped_scale": ("+= scale * acc_k;", "+= acc_k;"),
    "bwd_D_sign": ("Prow[j] * (dProw[j] - Di);", "Prow[j] * (dProw[j] + Di);"),
    "bwd_no_D": ("Prow[j] * (dProw[j] - Di);", "Prow[j] * dProw[j];"),
    "bwd_dv_from_ds": ("acc_v += P[(int64_t)i * s_k + j]", "acc_v += dP[(int64_t)i * s_k + j]"),
    "bwd_dk_from_p": ("acc_k += dP[(int64_t)i * s_k + j]", "acc_k += P[(int64_t)i * s_k + j]"),
    "bwd_dp_with_k": ("dot += dOb[(int64_t)i * qs + c] * Vb[", "dot += dOb[(int64_t)i * qs + c] * Kb["),
    "bwd_dq_with_v": ("acc += dSrow[j] * Kb[", "acc += dSrow[j] * Vb["),
    "bwd_mask_off_by_one": ("if (causal && j > i + off) Prow[j]", "if (causal && j >= i + off) Prow[j]"),
    "bwd_gqa_overwrites": ("dVb[(int64_t)j * ks + c] += acc_v;", "dVb[(int64_t)j * ks + c] = acc_v;"),
    # FP8 inputs
    "e4m3_bias_8": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_subnormal_scale": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "e4m3_mantissa_sixteenths": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 16.0, e - 7)"),
    "fp8_v_takes_k_scale": ("V[t] = v_scale * e4m3_to_double(v[t]);",
                            "V[t] = k_scale * e4m3_to_double(v[t]);"),
    "bwd_D_from_first_key": ("for (int j = 0; j < s_k; ++j) Di += Prow[j] * dProw[j];",
                             "for (int j = 0; j < 1; ++j) Di += Prow[j] * dProw[j];"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new, 1))
    so = tmp_path / "mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(mut), "-o", str(so), "-lm"],
                   check=True)
    bad = failing_pins(oracle.load(str(so)))
    assert bad, f"planted mistake '{name}' passed every pin"


# Planted mistakes in the oracle's packed-batch wrapper (Python): the
# function's source is rewritten, compiled in the oracle module's namespace
# and swapped in for the pins; each mutant must fail at least one pin.
VARLEN_MUTANTS = {
    "varlen_keys_at_query_offsets": ("kb[None, k0:k1], vb[None, k0:k1]",
                                     "kb[None, q0:q1], vb[None, q0:q1]"),
    "varlen_skips_last_sequence": ("for b in range(len(cu_q) - 1):",
                                   "for b in range(len(cu_q) - 2):"),
    "varlen_drops_window": ("window_left=window_left)", "window_left=-1)"),
    "varlen_lse_rows_reversed": ("lse[:, q0:q1] = lb[0]", "lse[:, q0:q1] = lb[0][:, ::-1]"),
    "varlen_heads_not_transposed": ("o[q0:q1] = ob[0].transpose(1, 0, 2)",
                                    "o[q0:q1] = ob[0].reshape(o[q0:q1].shape)"),
    "varlen_v_from_k": ("vb[None, k0:k1], causal", "kb[None, k0:k1], causal"),
}


def _rebuilt_varlen(old: str | None = None, new: str | None = None):
    """oracle.attn_fwd_varlen recompiled from its source, with `old`
    replaced by `new` (once) when given."""
    import inspect
    import textwrap

    src = textwrap.dedent(inspect.getsource(oracle.attn_fwd_varlen))
    if old is not None:
        assert src.count(old) == 1, f"mutation site {old!r} not found"
        src = src.replace(old, new)
    ns = dict(vars(oracle))
    exec(compile(src, "<varlen rebuilt>", "exec"), ns)  # noqa: S102
    return ns["attn_fwd_varlen"]


def test_rebuilt_varlen_passes_every_pin(lib, monkeypatch):
    """Control for the mutants below: the unmodified source, rebuilt the
    same way, fails no pin (so a mutant's failure is its mistake's)."""
    monkeypatch.setattr(oracle, "attn_fwd_varlen", _rebuilt_varlen())
    assert failing_pins(lib) == []


@pytest.mark.parametrize("name", sorted(VARLEN_MUTANTS))
def test_planted_varlen_mistake_is_caught(lib, monkeypatch, name):
    monkeypatch.setattr(oracle, "attn_fwd_varlen", _rebuilt_varlen(*VARLEN_MUTANTS[name]))
    bad = failing_pins(lib)
    assert bad, f"planted mistake '{name}' passed every pin"
