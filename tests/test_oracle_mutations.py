"""The oracle's pins catch plausible mistakes (no GPU).

A pin is only worth as much as the mistakes it would catch.  Each case below
plants one mistake in a copy of one oracle function -- a dropped term, a
flipped sign, an index or operand exchanged, a rounding or summation order
changed, a stream word or byte misplaced -- and runs the pin suite of
``tests/test_oracle_*.py`` against the mutated oracle: at least one pin must
fail.  The mistake is planted on the CPU, in the oracle's own source: the
function's text is edited (every edited snippet must occur exactly once, so a
later change to the oracle breaks the case loudly instead of silently turning
it into a no-op) and compiled in place of the original for the length of the
case, in every module that holds a reference to it.

Some readings cannot be pinned on the CPU at all: which stream tag an operand
draws from, or how the stream's values are laid over a tensor's elements, are
conventions the pages leave open; any choice passes every CPU pin and only the
bit-exact device comparison tells them apart.  What the CPU does pin is that
the operands draw separate streams (mean and residual, activation and
gradient, one expert and the next), and the cases that break that are here.

A control case runs the same harness on the unmodified oracle and requires
every pin to pass, so that a broken harness cannot pass the mutation cases.
"""

import inspect
import sys
import textwrap

import pytest

import oracle
from oracle import averis as A
from oracle import nvfp4 as N
from oracle import philox as P
from oracle import stats as S

import test_oracle_formats as tf
import test_oracle_moe as tm
import test_oracle_philox as tp
import test_oracle_split as ts
import test_oracle_stats as tst
import test_oracle_wgrad as tw


def _pins(mod, *skip):
    """Every test function of a pin module (parametrised ones once per
    parameter), except the named ones."""
    out = []
    for name, fn in vars(mod).items():
        if not name.startswith("test_") or name in skip or not callable(fn):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if marks:
            argname, values = marks[0].args[0], marks[0].args[1]
            out += [(f"{name}[{v}]", fn, {argname: v}) for v in values]
        else:
            out.append((name, fn, {}))
    return out


# The slow pins (seconds each) run only for the cases that name them.
SLOW = {
    "test_group_values_uniform_and_round_ups_uncorrelated": tp.test_group_values_uniform_and_round_ups_uncorrelated,
    "test_sr_is_unbiased_over_seeds": tp.test_sr_is_unbiased_over_seeds,
    "test_stochastic_wgrad_is_unbiased": tw.test_stochastic_wgrad_is_unbiased,
    "test_cos_mean_top_singular_vector": tst.test_cos_mean_top_singular_vector,
}

FAST_PINS = (_pins(tf) + _pins(tp, *SLOW) + _pins(ts) + _pins(tm) + _pins(tw, *SLOW) + _pins(tst, *SLOW))


def _mutant(module, name, edits):
    """Compile ``module.name`` with the textual edits applied, in a copy of
    the module's namespace."""
    src = textwrap.dedent(inspect.getsource(getattr(module, name)))
    for old, new in edits:
        assert src.count(old) == 1, f"{module.__name__}.{name}: snippet {old!r} found {src.count(old)} times"
        src = src.replace(old, new)
    ns = dict(vars(module))
    exec(compile(src, f"<planted mistake in {module.__name__}.{name}>", "exec"), ns)
    return ns[name]


def _plant(monkeypatch, module, name, edits):
    """Replace ``module.name`` by its mutant wherever a module holds it."""
    orig = getattr(module, name)
    mutant = _mutant(module, name, edits)
    for mod in list(sys.modules.values()):
        modname = getattr(mod, "__name__", "") or ""
        if not (modname == "oracle" or modname.startswith("oracle.") or modname.startswith("test_oracle_")):
            continue
        if getattr(mod, name, None) is orig:
            monkeypatch.setattr(mod, name, mutant)


def _run(pins, stop_at_first=True):
    """(name, exception) of every pin that failed."""
    failed = []
    for label, fn, kwargs in pins:
        try:
            fn(**kwargs)
        except Exception as e:            # an assertion, or an error the mistake provoked
            failed.append((label, e))
            if stop_at_first:
                break
    return failed


# (id, module, function, [(old, new), ...], slow pins that must fail as well)
MUTATIONS = [
    # ---- E2M1 ----
    ("e2m1_rne tie 1.25 rounds up", N, "e2m1_rne", [("(a > 1.25)", "(a >= 1.25)")], []),
    ("e2m1_rne tie 0.75 rounds down", N, "e2m1_rne", [("(a >= 0.75)", "(a > 0.75)")], []),
    ("e2m1_rne loses the sign of a zero", N, "e2m1_rne",
     [("sign = np.signbit(y).astype(np.uint8) << 3", "sign = (np.signbit(y) & (code > 0)).astype(np.uint8) << 3")], []),
    ("e2m1_sr carry off by one", N, "e2m1_sr", [("np.int64)) >= 65536", "np.int64)) > 65536")], []),
    ("e2m1_sr position measured from zero", N, "e2m1_sr", [("((a - lo) / step)", "(a / step)")], []),
    ("e2m1_sr drops the sign", N, "e2m1_sr", [("return (code | sign)", "return (code | 0 * sign)")], []),
    ("e2m1_value sign from bit 2", N, "e2m1_value", [("np.where(c & 8, -mag, mag)", "np.where(c & 4, -mag, mag)")], []),
    # ---- E4M3 ----
    ("e4m3_value exponent bias 8", N, "e4m3_value", [("np.exp2(e - 7.0)", "np.exp2(e - 8.0)")], []),
    ("e4m3_value subnormal as normal", N, "e4m3_value", [("np.where(e == 0, m", "np.where(e < 0, m")], []),
    ("e4m3_rne truncates", N, "e4m3_rne_satfinite", [("np.rint(sp / q)", "np.floor(sp / q)")], []),
    ("e4m3_rne ties away from zero", N, "e4m3_rne_satfinite", [("np.rint(sp / q)", "np.floor(sp / q + 0.5)")], []),
    ("e4m3_rne saturates to the NaN code", N, "e4m3_rne_satfinite",
     [("np.where(sat, 0x7E, code)", "np.where(sat, 0x7F, code)")], []),
    # ---- scale layout and packing ----
    ("scale_offset row and lane quarter exchanged", N, "scale_offset",
     [("(r % 32) * 16 + ((r % ATOM_ROWS) // 32) * 4", "(r % 32) * 4 + ((r % ATOM_ROWS) // 32) * 128")], []),
    ("scale_offset atoms column-group major", N, "scale_offset",
     [("(r // ATOM_ROWS) * n_kb64 + c // ATOM_COLS", "(c // ATOM_COLS) * n_kb64 + r // ATOM_ROWS")], []),
    ("pack_codes element 2k in the high nibble", N, "pack_codes",
     [("codes[:, 0::2] | (codes[:, 1::2] << 4)", "codes[:, 1::2] | (codes[:, 0::2] << 4)")], []),
    ("unpack_codes nibbles exchanged", N, "unpack_codes",
     [("out[:, 0::2] = packed & 0xF", "out[:, 0::2] = packed >> 4"),
      ("out[:, 1::2] = packed >> 4", "out[:, 1::2] = packed & 0xF")], []),
    # ---- the block quantizer ----
    ("tensor scale without the E2M1 maximum", N, "tensor_scales",
     [("np.float32(FP4_FP8_PRODUCT / A)", "np.float32(E4M3_MAX / A)")], []),
    ("block scale from a_b / 4", N, "nvfp4_quantize", [("(a_b / np.float32(6.0))", "(a_b / np.float32(4.0))")], []),
    ("block reciprocal inverted", N, "nvfp4_quantize",
     [("(g_enc / np.where(S == 0, 1.0, Sv))", "(np.where(S == 0, 1.0, Sv) / g_enc)")], []),
    ("blocks strided instead of contiguous", N, "nvfp4_quantize",
     [("blocks = T.reshape(R, K // BLOCK, BLOCK)", "blocks = T.reshape(R, BLOCK, K // BLOCK).transpose(0, 2, 1)")], []),
    ("dequantize without the tensor scale", N, "nvfp4_dequantize",
     [("return v * s * np.float64(q.g_dec)", "return v * s")], []),
    ("dequantize tiles the block scales", N, "nvfp4_dequantize",
     [("np.repeat(e4m3_value(q.scales).astype(np.float64), BLOCK, axis=1)",
       "np.tile(e4m3_value(q.scales).astype(np.float64), (1, BLOCK))")], []),
    # ---- Philox and the stream ----
    ("philox nine rounds", P, "philox4x32_10", [("range(10)", "range(9)")], []),
    ("philox multipliers exchanged", P, "philox4x32_10",
     [("p0 = M0 * c0", "p0 = M1 * c0"), ("p1 = M1 * c2", "p1 = M0 * c2")], []),
    ("philox second key word bumped by W0", P, "philox4x32_10",
     [("k1 = (k1 + W1) & MASK32", "k1 = (k1 + W0) & MASK32")], []),
    ("philox product halves exchanged", P, "philox4x32_10",
     [("(p1 >> SHIFT32) ^ c1 ^ k0, p1 & MASK32", "(p1 & MASK32) ^ c1 ^ k0, p1 >> SHIFT32")], []),
    ("counter words of the offset exchanged", P, "random_words",
     [("philox4x32_10(g & MASK32, g >> SHIFT32,", "philox4x32_10(g >> SHIFT32, g & MASK32,")], []),
    ("tag in the fourth counter word", P, "random_words",
     [("np.full_like(g, np.uint64(tag)), np.zeros_like(g),", "np.zeros_like(g), np.full_like(g, np.uint64(tag)),")], []),
    ("output words in reverse order", P, "random_words",
     [("words[(gi % np.uint64(4)).astype(np.int64)", "words[(np.uint64(3) - gi % np.uint64(4)).astype(np.int64)")], []),
    ("two elements of a group read the same bits", P, "group_values16",
     [("[W, _bitrev16(W), V, _bitrev16(V)]", "[W, _bitrev16(W), V, V]")],
     ["test_group_values_uniform_and_round_ups_uncorrelated"]),
    ("the first element's value reused by the third", P, "group_values16",
     [("[W, _bitrev16(W), V, _bitrev16(V)]", "[W, _bitrev16(W), W, _bitrev16(V)]")],
     ["test_group_values_uniform_and_round_ups_uncorrelated"]),
    ("a byte of the word read twice", P, "group_values16", [("W = (b2 << 8) | b0", "W = (b0 << 8) | b0")], []),
    # ---- the mean and the split ----
    ("rows added in reverse within a chunk", A, "column_mean",
     [("for i in range(c0, min(c0 + CHUNK, l)):", "for i in reversed(range(c0, min(c0 + CHUNK, l))):")], []),
    ("chunks added in reverse", A, "column_mean",
     [("for c0 in range(0, l, CHUNK):", "for c0 in reversed(range(0, l, CHUNK)):")], []),
    ("chunks of 128 rows", A, "column_mean",
     [("range(0, l, CHUNK)", "range(0, l, CHUNK // 2)"), ("min(c0 + CHUNK, l)", "min(c0 + CHUNK // 2, l)")], []),
    ("one running sum, no chunk partials", A, "column_mean",
     [("p = np.zeros(m, dtype=np.float32)", "p = S"), ("S = S + p", "S = p")], []),
    ("mean divides by l - 1", A, "column_mean", [("(S / np.float32(l))", "(S / np.float32(l - 1))")], []),
    ("split adds the mean", A, "mean_residual_split",
     [("(_as_f32(X) - np.asarray(mu, dtype=np.float32)[None, :])",
       "(_as_f32(X) + np.asarray(mu, dtype=np.float32)[None, :])")], []),
    ("residual amax taken of X", A, "column_mean_and_residual_amax",
     [("np.max(np.abs(XR))", "np.max(np.abs(_as_f32(X)))")], []),
    ("mean quantized from the residual's stream", A, "averis_split_quant",
     [("mu_q = nvfp4_quantize(mu[None, :], rounding, seed, offset, t_mu)",
       "mu_q = nvfp4_quantize(mu[None, :], rounding, seed, offset, t_r)")], []),
    ("gradient split on the activation's streams", A, "averis_split_quant",
     [("if grad else (TAGS[\"x_r\"], TAGS[\"mu_x\"])", "if False else (TAGS[\"x_r\"], TAGS[\"mu_x\"])")], []),
    ("mean quantized with the residual's tensor scale", A, "averis_split_quant",
     [("mu_q = nvfp4_quantize(mu[None, :], rounding, seed, offset, t_mu)",
       "mu_q = nvfp4_quantize(mu[None, :], rounding, seed, offset, t_mu, amax=A)")], []),
    # ---- the reference products ----
    ("gemm reference drops the bias", A, "gemm_reference",
     [("Y = Y + np.asarray(bias, dtype=np.float64)[None, :]", "Y = Y")], []),
    ("linear reference drops the rank-one row", A, "averis_linear_reference",
     [("return gemm_reference(xr_q, w_q, b)", "return gemm_reference(xr_q, w_q)")], []),
    # ---- the weight gradient ----
    ("wgrad drops the rank-one term", A, "wgrad_reference", [("float(l) * np.outer(", "0.0 * np.outer(")], []),
    ("wgrad rank-one term scaled by l - 1", A, "wgrad_reference", [("float(l) * np.outer(", "float(l - 1) * np.outer(")], []),
    ("token padding filled with ones", A, "transpose_padded",
     [("out = np.zeros((K, padded_tokens(l)), dtype=np.float32)", "out = np.ones((K, padded_tokens(l)), dtype=np.float32)")], []),
    ("token axis padded to 16", A, "padded_tokens",
     [("(int(l) + TOKEN_ALIGN - 1) // TOKEN_ALIGN * TOKEN_ALIGN", "(int(l) + 15) // 16 * 16")], []),
    # ---- MoE ----
    ("expert segments aligned to 64", A, "moe_offsets",
     [("(int(n) + MOE_ALIGN - 1) // MOE_ALIGN * MOE_ALIGN", "(int(n) + 63) // 64 * 64")], []),
    ("expert statistics from the buffer's start", A, "moe_split_quant", [("Xe = X[o:o + n]", "Xe = X[:o + n]")], []),
    ("every expert's stream starts at the offset", A, "moe_split_quant",
     [("offset + (o * K) // 16, t_r", "offset, t_r")], []),
    # ---- the monitor ----
    ("energy ratio normalised by the token count", S, "mean_energy_ratio", [("m = X.shape[1]", "m = X.shape[0]")], []),
    ("energy ratio without the square root", S, "mean_energy_ratio",
     [("math.sqrt(np.mean(np.sum(X * X, axis=1)) / m)", "(np.mean(np.sum(X * X, axis=1)) / m)")], []),
]


def test_control_every_pin_passes_on_the_unmodified_oracle():
    failed = _run(FAST_PINS + [(k, f, {}) for k, f in SLOW.items()], stop_at_first=False)
    assert not failed, failed
    assert len(FAST_PINS) >= 50


@pytest.mark.parametrize("case", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_a_planted_mistake_fails_a_pin(case, monkeypatch):
    _, module, name, edits, must_fail = case
    _plant(monkeypatch, module, name, edits)
    assert _run(FAST_PINS), f"no pin catches: {case[0]}"
    for pin in must_fail:
        assert _run([(pin, SLOW[pin], {})]), f"{pin} does not catch: {case[0]}"
