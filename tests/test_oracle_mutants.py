"""The pins are sensitive: plant plausible mistakes in a COPY of the oracle's C
source (on the CPU, in a temporary directory), rebuild it, and check that at
least one pin fails for every mutant. The committed oracle is not touched."""
import ctypes
import os
import subprocess

import pytest

import oracle

from . import test_oracle_backward as bw
from . import test_oracle_cells as cells
from . import test_oracle_pins as pins

# (name, original text, mutated text) -- each replacement must hit exactly once
MUTANTS = [
    ("flipped_orientation", "const int ih = oh * f->stride + kh - f->pad;",
     "const int ih = oh * f->stride + (f->KH - 1 - kh) - f->pad;"),
    ("swapped_kh_kw", "(((size_t)co * f->KH + kh) * f->KW + kw) * Cg",
     "(((size_t)co * f->KH + kw) * f->KW + kh) * Cg"),
    ("dropped_bias", "double s = bb[co];", "double s = 0.0;"),
    ("alpha_transposed", "const double *ab = f->alpha + (size_t)b * f->n;",
     "const double *ab = f->alpha + (size_t)b;"),
    ("wrong_group_offset", "* f->Cin + (size_t)g * Cg;", "* f->Cin + (size_t)0 * Cg;"),
    ("gap_not_averaged", "g[c] = s / (double)(H * W);", "g[c] = s;"),
    ("softmax_without_tau", "den += exp(z[j] / tau);", "den += exp(z[j]);"),
    ("router_bias_dropped", "double s = br ? br[i] : 0.0;", "double s = 0.0;"),
    ("sign_error_in_sigmoid", "1.0 / (1.0 + exp(-z[i]))", "1.0 / (1.0 + exp(z[i]))"),
    ("stride_ignored_in_w", "const int iw = ow * f->stride + kw - f->pad;",
     "const int iw = ow + kw - f->pad;"),
    ("input_attention_on_wrong_channel", "for (int ci = 0; ci < Cg; ++ci) s += (ap[ci] * xp[ci]) * wp[ci];",
     "for (int ci = 0; ci < Cg; ++ci) s += (ap[Cg - 1 - ci] * xp[ci]) * wp[ci];"),
    ("output_attention_before_bias", "double s = bb[co];", "double s = aout ? bb[co] / aout[co] : bb[co];"),
    ("output_attention_dropped", "if (aout) s *= aout[co];", "if (0) s *= aout[co];"),
    # backward
    ("sigmoid_grad_missing_factor", "dz[i] = da[i] * a[i] * (1.0 - a[i]);", "dz[i] = da[i] * a[i];"),
    ("softmax_grad_missing_tau", "dz[i] = a[i] * (da[i] - dot) / tau;",
     "dz[i] = a[i] * (da[i] - dot);"),
    ("softmax_grad_not_centred", "dz[i] = a[i] * (da[i] - dot) / tau;", "dz[i] = a[i] * da[i] / tau;"),
    ("pool_grad_not_averaged", "dxb[(size_t)p * f->Cin + c] += dgb[c] * inv;",
     "dxb[(size_t)p * f->Cin + c] += dgb[c];"),
    ("pool_grad_dropped", "if (f->dg) {", "if (0) {"),
    ("dalpha_bias_term_dropped",
     "s += db[(size_t)b * Cout + co] * bias[(size_t)i * Cout + co];",
     "s += 0.0 * db[(size_t)b * Cout + co];"),
    ("dexperts_wrong_expert",
     "for (int b = 0; b < B; ++b) s += alpha[(size_t)b * n + i] * dW[(size_t)b * wsize + e];",
     "for (int b = 0; b < B; ++b) s += alpha[(size_t)b * n + (n - 1 - i)] * dW[(size_t)b * wsize + e];"),
    ("dbias_without_alpha",
     "for (int b = 0; b < B; ++b) s += alpha[(size_t)b * n + i] * db[(size_t)b * Cout + co];",
     "for (int b = 0; b < B; ++b) s += db[(size_t)b * Cout + co];"),
    ("weight_grad_channel_reversed", "for (int ci = 0; ci < Cg; ++ci) gw[ci] += d * xp[ci];",
     "for (int ci = 0; ci < Cg; ++ci) gw[ci] += d * xp[Cg - 1 - ci];"),
    ("data_grad_kernel_flipped",
     "const double *wv = Wb + ((size_t)(co * f->KH + kh) * f->KW + kw) * Cg;",
     "const double *wv = Wb + ((size_t)(co * f->KH + (f->KH - 1 - kh)) * f->KW + (f->KW - 1 - kw)) * Cg;"),
    ("weight_grad_stride_ignored",
     "const int y_in = f->stride * oh - f->pad + kh, x_in = f->stride * ow - f->pad + kw;\n"
     "            if (y_in < 0 || y_in >= f->H || x_in < 0 || x_in >= f->W) continue;  /* padding */\n"
     "            const double *xp",
     "const int y_in = oh - f->pad + kh, x_in = ow - f->pad + kw;\n"
     "            if (y_in < 0 || y_in >= f->H || x_in < 0 || x_in >= f->W) continue;  /* padding */\n"
     "            const double *xp"),
    ("router_weight_grad_uses_dalpha",
     "for (int c = 0; c < C; ++c) dWr[(size_t)i * C + c] += dz[i] * g[c];",
     "for (int c = 0; c < C; ++c) dWr[(size_t)i * C + c] += da[i] * g[c];"),
    ("pool_grad_wrong_router_row", "for (int i = 0; i < n; ++i) s += dz[i] * Wr[(size_t)i * C + c];",
     "for (int i = 0; i < n; ++i) s += dz[i] * Wr[(size_t)(n - 1 - i) * C + c];"),
    # kernel cells
    ("cells_share_first_cells_attention", "acc += alpha_b[(size_t)j * n + i] * warehouse[(size_t)i * s + e];",
     "acc += alpha_b[i] * warehouse[(size_t)i * s + e];"),
    ("cells_written_over_each_other", "Wb[(size_t)j * s + e] = acc;", "Wb[e] = acc;"),
    ("cells_activation_on_first_block", "oracle_act(n, z + (size_t)j * n, mode, tau,",
     "oracle_act(n, z, mode, tau,"),
]

PIN_TESTS = [
    lambda: [pins.test_n1_alpha1_is_static_conv_torch(s) for s in pins.SHAPES],
    lambda: [pins.test_mixed_kernel_matches_torch_conv(s) for s in pins.SHAPES],
    lambda: [pins.test_brute_force_second_formulation(s) for s in range(12)],
    pins.test_impulse_pins_orientation,
    pins.test_zero_input_gives_mixed_bias_and_route_of_br,
    pins.test_constant_input_route_closed_form,
    lambda: [pins.test_route_against_library_routines(m, t)
             for m, t in [(0, 1.0), (1, 1.0), (1, 0.3), (1, 30.0)]],
    pins.test_route_invariants,
    lambda: [pins.test_channel_attention_matches_torch_conv(s) for s in pins.SHAPES],
    pins.test_channel_attention_zero_input_gives_scaled_bias,
    # backward
    lambda: [bw.test_central_differences_every_input(c) for c in bw.CASES],
    lambda: [bw.test_central_differences_attention_as_input(c) for c in bw.CASES[:4]],
    lambda: [bw.test_matches_torch_autograd(c) for c in bw.CASES],
    bw.test_softmax_router_gradients_sum_to_zero_over_experts,
    bw.test_zero_input_leaves_bias_terms,
    bw.test_pooled_gradient_adds_a_constant_per_channel,
    # kernel cells
    lambda: [cells.test_one_hot_attentions_pick_whole_cells(sh) for sh in cells.SHAPES],
    lambda: [cells.test_cell_routing_is_the_routing_per_cell(m, t)
             for m, t in [(0, 1.0), (1, 1.0), (1, 3.0)]],
    cells.test_a_cell_changes_only_its_output_channels,
]


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, orig, mut):
    src = open(oracle._SRC).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not unique"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(orig, mut))
    so = tmp_path / "mutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", str(path_c),
                    "-o", str(so), "-lm"], check=True)
    saved = oracle._lib
    oracle._lib = oracle.configure(ctypes.CDLL(str(so)))
    failures = 0
    try:
        for t in PIN_TESTS:
            try:
                t()
            except (AssertionError, ValueError):
                failures += 1
                break  # one failing pin is enough
    finally:
        oracle._lib = saved
    assert failures > 0, f"no pin caught mutant {name}"
