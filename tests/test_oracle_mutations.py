"""Planted-mistake check for the oracle's pins (CPU only).

Each case copies oracle/rodref.c to a temporary directory, plants one plausible mistake by a
textual substitution (a gate applied to the wrong channel, a decay that also hits the new
term, the readout using k, an off-by-one window, a dropped scale or normaliser, a wrong
ring-buffer slot, a hand-off that drops a token or numbers slots from the window start, a paged cache read
without its table or written at the wrong row, a backward that weights the gate gradient
with the updated state or decays the gradient state on the wrong channel, an attention backward
without the softmax row term or with the shared key's gradient from one head, a row log-sum-exp
without its maximum, an E4M3 encoder
that breaks ties to the odd code, misplaces the subnormals or does not saturate, an FP8 decode
that forgets the value scale, an FP8 fill that multiplies by the scale), builds the copy with gcc and runs every pin against it. Each planted
mistake must make at least one pin fail; otherwise the pins are too weak to trust.
"""
import inspect
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import build as obuild

from . import test_oracle_pins as pins
from . import test_oracle_swska_lse as lse_pins

MUTATIONS = {
    "gate_on_wrong_channel": ("const double gc = (double)g[c];",
                              "const double gc = (double)g[(c + 1) % dk];"),
    "decay_hits_new_term": ("row[j] = gc * row[j] + kc * (double)v[j];",
                            "row[j] = gc * (row[j] + kc * (double)v[j]);"),
    "readout_uses_key": ("acc += (double)q[c] * S[c * dv + j];",
                         "acc += (double)k[c] * S[c * dv + j];"),
    "window_one_too_wide": ("int64_t j0 = t - a->W + 1;", "int64_t j0 = t - a->W;"),
    "scale_dropped": ("s[j - j0] = scale * acc;", "s[j - j0] = acc;"),
    "normaliser_dropped": ("for (int64_t i = 0; i < dv; ++i) out[i] /= l;\n    return m + log(l);\n}",
                           "for (int64_t i = 0; i < dv; ++i) out[i] /= 1.0;\n    return m + log(l);\n}"),
    "lse_without_max": ("    return m + log(l);\n}", "    return log(l);\n}"),
    "ring_slot_off_by_one": ("const int64_t slot = pos[n] % W;",
                             "const int64_t slot = (pos[n] + 1) % W;"),
    "decode_window_too_wide": ("const int64_t p0 = P - a->W + 1 > 0 ? P - a->W + 1 : 0;",
                               "const int64_t p0 = P - a->W > 0 ? P - a->W : 0;"),
    "cache_fill_drops_oldest": ("const int64_t p0 = T > W ? T - W : 0;",
                                "const int64_t p0 = T > W ? T - W + 1 : 0;"),
    "cache_fill_slot_from_start": ("const int64_t slot = p % W;",
                                   "const int64_t slot = (p - p0) % W;"),
    "paged_read_ignores_table": ("const int64_t t = table[n * pps + s / page], r = s % page;",
                                 "const int64_t t = n * pps + s / page, r = s % page;"),
    "bwd_dg_with_new_state": ("accg += dS[c * dv + j] * Sprev[c * dv + j];",
                              "accg += dS[c * dv + j] * Sprev[DD + c * dv + j];"),
    "bwd_decay_wrong_channel": ("for (int64_t j = 0; j < dv; ++j) dS[c * dv + j] *= (double)a->g[tk + c];",
                                "for (int64_t j = 0; j < dv; ++j) dS[c * dv + j] *= (double)a->g[tk + (c + 1) % dk];"),
    "ska_bwd_drops_row_term": ("const double dS = pr[j - j0] * (dp[j - j0] - D);",
                               "const double dS = pr[j - j0] * dp[j - j0];"),
    "ska_bwd_shared_key_one_head": ("for (int64_t h = 0; h < H; ++h) acc += dkp[(b * H + h) * T * dk + i];",
                                    "for (int64_t h = 0; h < 1; ++h) acc += dkp[(b * H + h) * T * dk + i];"),
    "paged_write_wrong_row": ("t = table[n * pps + s / page], r = s % page;\n            memcpy(k_pool",
                              "t = table[n * pps + s / page], r = (s + 1) % page;\n            memcpy(k_pool"),
    "e4m3_ties_to_odd": ("best = dl < dh ? lo : (dh < dl ? hi : ((lo & 1) == 0 ? lo : hi));",
                         "best = dl < dh ? lo : (dh < dl ? hi : ((lo & 1) == 1 ? lo : hi));"),
    "e4m3_subnormal_exponent": ("v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    "e4m3_no_saturation": ("    if (a >= 448.0) {\n        best = 0x7E;", "    if (a >= 464.0) {\n        best = 0x7F;"),
    "fp8_decode_v_unscaled": ("on[c] += s[i] * e4m3_table[a->vc[((n * H + h) * W + sl) * dv + c]] * a->v_scale;",
                              "on[c] += s[i] * e4m3_table[a->vc[((n * H + h) * W + sl) * dv + c]];"),
    "fp8_fill_scale_multiplies": ("k_cache[(b * W + ring_slot) * dk + c] = rodref_e4m3_encode(k[(b * T + p) * dk + c] / k_scale);",
                                  "k_cache[(b * W + ring_slot) * dk + c] = rodref_e4m3_encode(k[(b * T + p) * dk + c] * k_scale);"),
}


def _pin_calls():
    """Every pin test with each of its parametrizations, as zero-argument callables."""
    calls = []
    for name, fn in [m for mod in (pins, lse_pins) for m in inspect.getmembers(mod, inspect.isfunction)]:
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            calls.append((name, fn, {}))
            continue
        argnames, values = params[0].args[0], params[0].args[1]
        names = [a.strip() for a in argnames.split(",")]
        for val in values:
            val = val if len(names) > 1 else (val,)
            calls.append((name, fn, dict(zip(names, val))))
    return calls


def _build_mutant(tmp_path, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique/found: {old!r}"
    path = tmp_path / "rodref_mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "librodref_mut.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-o", str(so), str(path),
                    "-lm", "-lpthread"], check=True)
    return oracle.OracleLib(str(so))


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(mutation, tmp_path):
    old, new = MUTATIONS[mutation]
    lib = _build_mutant(tmp_path, old, new)
    caught = []
    with oracle.using(lib):
        for name, fn, kw in _pin_calls():
            try:
                fn(**kw)
            except AssertionError:
                caught.append(name)
    assert caught, f"no pin caught the planted mistake '{mutation}'"


def test_unmutated_copy_passes_every_pin(tmp_path):
    lib = _build_mutant(tmp_path, "int rodref_abi_version(void) { return 1; }",
                        "int rodref_abi_version(void) { return 1; }")
    with oracle.using(lib):
        for name, fn, kw in _pin_calls():
            fn(**kw)
