"""Plant plausible mistakes in copies of the oracle and check that the pins
catch every one of them.  Each mutant is the oracle's C source with one text
substitution, compiled into a temporary library (the oracle itself is never
modified)."""
import os

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_ref.c")

# (name, original text, mutated text) -- each original must occur in the source
MUTANTS = [
    ("h0 ignored", "h[n] = a->h0 ? (double)a->h0[chan * N + n] : 0.0;", "h[n] = 0.0;"),
    ("A sign flipped", "exp(dt * (double)a->A[d * N + n])", "exp(-dt * (double)a->A[d * N + n])"),
    ("Euler term without dt", "h[n] = abar * h[n] + dt * bt * xt;", "h[n] = abar * h[n] + bt * xt;"),
    ("ZOH uses exp(A) not exp(dt A)", "exp(dt * (double)a->A[d * N + n])", "exp((double)a->A[d * N + n])"),
    ("D skip dropped", "y += (double)a->D[d] * xt;", "y += 0.0;"),
    ("gate is sigmoid not silu", "return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    ("softplus dropped", "const double dt = a->softplus ? softplus_ref(v) : v;", "const double dt = v;"),
    ("bias ignored", "v += (double)a->delta_bias[d];", "v += 0.0;"),
    ("softplus sign", "return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v)));",
     "return (v > 0.0 ? v : 0.0) + log1p(exp(fabs(v)));"),
    ("B and C swapped", "y += load_act(a->C, (b * N + n) * L + t, a->dtype) * h[n];",
     "y += load_act(a->B, (b * N + n) * L + t, a->dtype) * h[n];"),
    ("B read transposed [b][t][n]", "load_act(a->B, (b * N + n) * L + t, a->dtype);",
     "load_act(a->B, (b * L + t) * N + n, a->dtype);"),
    ("x read one step late", "const double xt = xrow ? xrow[t] : load_act(a->x, chan * L + t, a->dtype);",
     "const double xt = xrow ? xrow[t] : load_act(a->x, chan * L + (t + 1 < L ? t + 1 : t), a->dtype);"),
    ("C readout dropped", "        double y = 0.0;\n        for (int64_t n = 0; n < N; n++)\n            y += load_act(a->C",
     "        double y = 0.0;\n        for (int64_t n = 0; n < N; n++)\n            y += 0.0 * load_act(a->C"),
    ("state decays twice", "h[n] = abar * h[n] + dt * bt * xt;", "h[n] = abar * abar * h[n] + dt * bt * xt;"),
    ("A indexed [n][d]", "exp(dt * (double)a->A[d * N + n])", "exp(dt * (double)a->A[(n * a->dim + d) % (a->dim * N)])"),
    ("h_last returns the initial state", "            hl[n] = h[n];",
     "            hl[n] = a->h0 ? (double)a->h0[chan * N + n] : 0.0;"),
    ("step ignores gate", "            y *= silu_ref(load_act(z, c, dtype));", "            y *= 1.0;"),
    ("channel index b/d swapped", "scan_channel(&a, c / dim, c % dim,", "scan_channel(&a, c % batch, c / batch,"),
    # the causal convolution in front of the scan
    ("conv taps reversed", "acc += (double)w[d * K + k] * conv_input(",
     "acc += (double)w[d * K + (K - 1 - k)] * conv_input("),
    ("conv state ignored", "    if (!conv_state)\n        return 0.0;", "    if (1)\n        return 0.0;"),
    ("conv window one step late", "conv_input(x, conv_state, dtype, chan, L, K, t - K + 1 + k);",
     "conv_input(x, conv_state, dtype, chan, L, K, t - K + k);"),
    ("conv bias dropped", "        double acc = bias ? (double)bias[d] : 0.0;\n        for (int64_t k = 0; k < K; k++)",
     "        double acc = 0.0;\n        for (int64_t k = 0; k < K; k++)"),
    ("conv output not activated", "conv_channel(x, w, cbias, K, conv_state, 1, dtype,",
     "conv_channel(x, w, cbias, K, conv_state, 0, dtype,"),
    ("conv scan reads raw x", "scan_channel_x(&a, c / dim, c % dim, xc,", "scan_channel_x(&a, c / dim, c % dim, NULL,"),
    ("new conv state one input early", "conv_input(x, conv_state, dtype, chan, L, K, L - (K - 1) + j);",
     "conv_input(x, conv_state, dtype, chan, L, K, L - K + j);"),
    ("conv step does not shift", "            cs[k] = cs[k + 1];", "            cs[k] = cs[k];"),
    ("conv step window reversed", "acc += (double)w[d * K + k] * cs[k];", "acc += (double)w[d * K + k] * cs[K - 2 - k];"),
    # the exponential-trapezoidal rule
    ("trap weights swapped", "const double beta = (1.0 - lt) * dt * alpha;", "const double beta = lt * dt * alpha;"),
    ("trap start term not decayed", "const double beta = (1.0 - lt) * dt * alpha;",
     "const double beta = (1.0 - lt) * dt;"),
    ("trap end weight without dt", "const double gamma = lt * dt;", "const double gamma = lt;"),
    ("trap previous input never moves on", "            vprev[n] = vt;", "            vprev[n] = vprev[n];"),
    ("trap input before t = 0 ignored", "const double xp = (x_prev && B_prev) ? load_act(x_prev, chan, a->dtype) : 0.0;",
     "const double xp = 0.0;"),
    ("trap step mixes by 1 - lambda twice", "hl[n] = alpha * h[n] + (1.0 - lt) * dt * alpha * vprev[n] + lt * dt * vt;",
     "hl[n] = alpha * h[n] + (1.0 - lt) * dt * alpha * vprev[n] + (1.0 - lt) * dt * vt;"),
    # the backward pass
    ("bwd silu derivative wrong", "dz[chan * L + t] = go * y * s * (1.0 + zt * (1.0 - s));",
     "dz[chan * L + t] = go * y * s * (1.0 + zt * s);"),
    ("bwd adjoint not decayed", "            gnext_decayed[n] = abar * g[n];", "            gnext_decayed[n] = g[n];"),
    ("bwd dB without dt", "dB[(b * N + n) * L + t] += g[n] * dt * xt;", "dB[(b * N + n) * L + t] += g[n] * xt;"),
    ("bwd ddt drops the decay term", "ddt += g[n] * (An * abar * hp[n] + Bn * xt);", "ddt += g[n] * (Bn * xt);"),
    ("bwd dA uses h_t", "dA[d * N + n] += g[n] * dt * abar * hp[n];", "dA[d * N + n] += g[n] * dt * abar * ht[n];"),
    ("bwd softplus derivative dropped", "const double ddel = a->softplus ? ddt * sigmoid_ref(v) : ddt;",
     "const double ddel = ddt;"),
    ("bwd dx drops the skip", "double dxt = a->D ? (double)a->D[d] * dy : 0.0;", "double dxt = 0.0;"),
    ("bwd dC uses h_{t-1}", "dC[(b * N + n) * L + t] += dy * ht[n];", "dC[(b * N + n) * L + t] += dy * hp[n];"),
    ("bwd dh_last ignored", "gnext_decayed[n] = dh_last ? (double)dh_last[chan * N + n] : 0.0;",
     "gnext_decayed[n] = 0.0;"),
    # Mamba-2 SSD
    ("ssd decay applied after the input", "S[p * N + n] = at * S[p * N + n] + dtt * xp * Bn;",
     "S[p * N + n] = at * (S[p * N + n] + dtt * xp * Bn);"),
    ("ssd input without dt", "S[p * N + n] = at * S[p * N + n] + dtt * xp * Bn;",
     "S[p * N + n] = at * S[p * N + n] + xp * Bn;"),
    ("ssd wrong group of B and C", "const int64_t b = bh / Hh, h = bh % Hh, g = h / (Hh / G);",
     "const int64_t b = bh / Hh, h = bh % Hh, g = h % G;"),
    ("ssd readout dropped", "                    yp += S[p * N + n] * Cn;\n",
     "                    yp += 0.0;\n"),
    ("ssd skip dropped", "                    yp += (double)D[h] * xp;", "                    yp += 0.0;"),
    ("trap step drops the previous token", "hl[n] = alpha * h[n] + (1.0 - lt) * dt * alpha * vprev[n] + lt * dt * vt;",
     "hl[n] = alpha * h[n] + lt * dt * vt;"),
]


def _mutant(tmp_path, i, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutant {i}: text not found"
    msrc = src.replace(old, new)
    c_path = tmp_path / f"mut{i}.c"
    c_path.write_text(msrc)
    so = str(tmp_path / f"libmut{i}.so")
    oracle.build(force=True, src=str(c_path), out=so)
    return oracle.load(so)


@pytest.mark.parametrize("i", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, i):
    name, old, new = MUTANTS[i]
    orc = _mutant(tmp_path, i, old, new)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant '{name}' passed every pin"
