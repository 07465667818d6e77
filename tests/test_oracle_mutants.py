"""The pins must catch plausible mistakes in the oracle.

Each case copies the oracle's C source to a temporary directory, plants one
mistake by text replacement (a dropped term, a wrong sign, a wrong index, a
conjugate, a transposed layout), compiles it on the CPU and runs every pin
against it: at least one pin has to fail.  The committed oracle is untouched.
"""
import os

import pytest

import oracle
import pins

MUTANTS = {
    "drop_D_real": ("yt[p] = acc + (D ? D[h] * xt[p] : 0.0);", "yt[p] = acc;"),
    "decay_sign": ("const double a = exp(d * A[h]); /* one step of decay */",
                   "const double a = exp(-d * A[h]);"),
    "no_dt_on_input": ("double s = a * S[IDX2(p, n, dstate)] + d * xt[p] * Bt[n];",
                       "double s = a * S[IDX2(p, n, dstate)] + xt[p] * Bt[n];"),
    "readout_before_injection": ("acc += Ct[n] * s;\n                    }\n                    yt[p] = acc + (D",
                                 "acc += Ct[n] * (s - d * xt[p] * Bt[n]);\n                    }\n                    yt[p] = acc + (D"),
    "interleaved_groups": ("const long g = h / heads_per_group;\n            /* initial state",
                           "const long g = h % ngroups;\n            /* initial state"),
    "init_ignored": ("S[IDX2(p, n, dstate)] = init_state ? init_state[si] : 0.0;",
                     "S[IDX2(p, n, dstate)] = 0.0;"),
    "final_transposed": ("final_state[((size_t)(b * nheads + h) * headdim + p) * dstate + n] =",
                         "final_state[((size_t)(b * nheads + h) * dstate + n) * headdim + p] ="),
    "complex_conj_readout": ("acc += Ct[n] * s;\n                    }\n                    yt[p] = creal(acc)",
                             "acc += conj(Ct[n]) * s;\n                    }\n                    yt[p] = creal(acc)"),
    "complex_rotation_sign": ("const double complex a = cexp(d * Ac[h]);\n                const double *xt",
                              "const double complex a = cexp(d * conj(Ac[h]));\n                const double *xt"),
    "complex_imag_readout": ("yt[p] = creal(acc) +", "yt[p] = cimag(acc) +"),
    "decode_no_dt": ("Sp[n] = a * Sp[n] + d * xb[p] * Bb[n];", "Sp[n] = a * Sp[n] + xb[p] * Bb[n];"),
    "decode_complex_no_decay": ("Sp[n] = a * Sp[n] + (d * xb[p]) * Bb[n];",
                                "Sp[n] = Sp[n] + (d * xb[p]) * Bb[n];"),
    # the adjoint (gradient) oracle
    "bwd_ddt_no_decay_term": ("ddt[tb * nheads + h] = ddt_in + ga * A[h] * a;", "ddt[tb * nheads + h] = ddt_in;"),
    "bwd_dA_no_dt": ("dA[h] += ga * d * a;", "dA[h] += ga * a;"),
    "bwd_adjoint_not_decayed": ("Gs[i] *= a;    /* gradient", "Gs[i] *= 1.0;    /* gradient"),
    "bwd_dC_previous_state": ("dCt[n] += dyt[p] * ht[IDX2(p, n, dstate)];", "dCt[n] += dyt[p] * hp[IDX2(p, n, dstate)];"),
    "bwd_dB_overwritten": ("dBt[n] += d * xt[p] * Gs[IDX2(p, n, dstate)];", "dBt[n] = d * xt[p] * Gs[IDX2(p, n, dstate)];"),
    "bwd_complex_decay_not_conjugated": ("Gs[i] *= conj(a);", "Gs[i] *= a;"),
    "bwd_complex_dA_not_conjugated": ("dAc[h] += d * conj(a) * ga;", "dAc[h] += d * a * ga;"),
    "bwd_complex_dC_not_conjugated": ("dCt[n] += dyt[p] * conj(ht[IDX2(p, n, dstate)]);",
                                      "dCt[n] += dyt[p] * ht[IDX2(p, n, dstate)];"),
    "bwd_complex_readout_not_conjugated": ("Gs[IDX2(p, n, dstate)] += conj(Ct[n]) * dyt[p];",
                                           "Gs[IDX2(p, n, dstate)] += Ct[n] * dyt[p];"),
    "bwd_complex_ddt_imag_part": ("creal(ga * conj(Ac[h] * a))", "cimag(ga * conj(Ac[h] * a))"),
    "bwd_complex_input_grad_imag_part": ("rp += creal(conj(Bt[n]) * Gs", "rp += cimag(conj(Bt[n]) * Gs"),
    # the variants
    "conv_kernel_reversed": ("v += w[c * width + k] * u;", "v += w[c * width + (width - 1 - k)] * u;"),
    "conv_not_causal": ("const long s = t - (width - 1) + k;", "const long s = t + k;"),
    "conv_init_reversed": ("init[(b * channels + c) * (width - 1) + (width - 1) + s]",
                           "init[(b * channels + c) * (width - 1) - 1 - s]"),
    "conv_silu_sign": ("if (silu) v = v / (1.0 + exp(-v));", "if (silu) v = v / (1.0 + exp(v));"),
    "selective_A_first_state": ("h[n] = exp(step * A[d * dstate + n]) * h[n] + step * B[bc] * u;",
                                "h[n] = exp(step * A[d * dstate]) * h[n] + step * B[bc] * u;"),
    "selective_readout_before_update": ("                    acc += C[bc] * h[n];",
                                        "                    acc += C[bc] * (h[n] - step * B[bc] * u);"),
    "selective_group_modulo": ("const long g = d / (channels / ngroups);\n            for (long n = 0; n < dstate; ++n)\n                h[n] = init_state",
                               "const long g = d % ngroups;\n            for (long n = 0; n < dstate; ++n)\n                h[n] = init_state"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    find, repl = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(find) == 1, f"mutation site for {name} not found exactly once"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(find, repl))
    so = oracle.build(force=True, src=str(mut_src), out=str(tmp_path / "libmutant.so"))
    lib = oracle.load(so)
    failed = []
    for pin_name, pin in pins.all_pins():
        try:
            err = pin(lib)
        except Exception as exc:  # a crash of the mutant also counts as caught
            failed.append((pin_name, repr(exc)))
            continue
        if not err <= pins.PIN_TOL:
            failed.append((pin_name, err))
    assert failed, f"no pin caught mutant {name}"
