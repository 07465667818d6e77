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
