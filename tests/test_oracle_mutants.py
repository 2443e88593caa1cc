"""The oracle's pins have teeth: plausible mistakes planted into a copy of
the oracle's C source (a dropped term, a wrong sign, a transposed operand, a
wrong index or layer) must each make at least one pin fail.

Each case patches one expression of oracle/reann_oracle.c (or several, for a
mistake made consistently in the forward and the reverse sweep, which finite
differences cannot see), compiles the copy,
routes the oracle through it and runs an existing pin test expecting an
AssertionError.  The real oracle is restored afterwards.  Everything here is
CPU only.
"""
import os

import pytest

import oracle
import test_oracle_density as dens
import test_oracle_forces as forc
import test_oracle_md as md
import test_oracle_pair_density as pairden
import test_oracle_pairs as pairs

MUTANTS = [
    ("multinomial weight dropped",
     "return factorial(t[0] + t[1] + t[2]) / (factorial(t[0]) * factorial(t[1]) * factorial(t[2]));",
     "return 1.0;",
     lambda: dens.test_density_matches_multinomial_formula_every_layer("ag256")),
    ("force on the centre with the wrong sign",
     "gx[i * 3 + a] -= V[a];", "gx[i * 3 + a] += V[a];",
     lambda: forc.test_zero_net_force("ag256")),
    ("second hidden layer transposed",
     "(double)v->W2[(int64_t)h * H1 + k] * a1[k]", "(double)v->W2[(int64_t)k * H1 + h] * a1[k]",
     lambda: dens.test_t1_energy_is_the_local_eann_network_on_closed_form_density()),
    ("feature index (n, l) swapped",
     "coef[j * D + tuple_l(tau) * NP + nn]", "coef[j * D + nn * 3 + tuple_l(tau)]",
     lambda: dens.test_dimer_closed_form(2.9)),
    ("cutoff derivative dropped",
     "double dfc = -0.5 * (pi / c->r_cut) * sin(pi * r / c->r_cut);", "double dfc = 0.0;",
     lambda: forc.test_forces_match_central_differences("ag256", 10)),
    ("minimum image dropped",
     "v = v - box[a] * rint(v / box[a]);", "v = v;",
     lambda: pairs.test_fcc_shell_counts(4.09, 6.0, 78, 54)),
    ("energy read from the wrong layer",
     "&rho[((T - 1) * n + i) * DR], a1, a2, &Ei[i]", "&rho[((T > 1 ? T - 2 : 0) * n + i) * DR], a1, a2, &Ei[i]",
     lambda: forc.test_receptive_field_is_T_hops(2)),
    ("tanh derivative wrong",
     "g2[k] = s * (1.0 - a2[k] * a2[k]);", "g2[k] = s * (1.0 - a2[k]);",
     lambda: forc.test_forces_match_central_differences("water", 10)),
    ("input standardisation dropped in the backward",
     "gx[f] = s / (double)v->scale[f];", "gx[f] = s;",
     lambda: forc.test_forces_match_central_differences("hea", 10)),
    ("pair form: diagonal factor 2 dropped in the backward",
     "s += (mm == nn ? 2.0 : 1.0) * At[i * nA + mm * ntau + tau] *", "s += 1.0 * At[i * nA + mm * ntau + tau] *",
     lambda: pairden.test_pair_forces_match_central_differences()),
    ("thermostat: coupling factor (1 - c) dropped from the cross term",
     "sqrt(cc * (1.0 - cc) * K * Kt / Nf)", "sqrt(cc * K * Kt / Nf)",
     lambda: md.test_nvt_without_coupling_is_nve()),
    ("thermostat: cross term halved",
     "2.0 * R1 * sqrt(cc * (1.0 - cc) * K * Kt / Nf)", "1.0 * R1 * sqrt(cc * (1.0 - cc) * K * Kt / Nf)",
     lambda: md.test_nvt_kinetic_energy_is_canonical()),
    ("thermostat: work accumulated with the wrong sign",
     "W += Kn - K;", "W -= Kn - K;",
     lambda: md.test_nvt_effective_energy_is_conserved()),
    ("coefficient networks applied in reversed layer order (forward and backward)",
     ("&w.coef[t * c->n_elements + types[i]]", "&w.coef[(t - 1) * c->n_elements + types[i]]"),
     ("&w.coef[(T - 2 - t) * c->n_elements + types[i]]", "&w.coef[(T - 1 - t) * c->n_elements + types[i]]"),
     lambda: dens.test_message_passing_dimer_chain(3, (0, 1))),
    ("element 0's coefficient network used for every atom (forward and backward)",
     ("&w.coef[t * c->n_elements + types[i]]", "&w.coef[(t - 1) * c->n_elements + types[i]]"),
     ("&w.coef[t * c->n_elements + 0]", "&w.coef[(t - 1) * c->n_elements + 0]"),
     lambda: dens.test_message_passing_dimer_chain(2, (0, 1))),
    ("coefficient network chosen by the neighbour's element",
     "&w.coef[t * c->n_elements + types[i]]", "&w.coef[t * c->n_elements + types[n - 1 - i]]",
     lambda: dens.test_message_passing_dimer_chain(2, (0, 1))),
    ("pair form: second factor taken from the same radial index",
     "tuple_weight(tau) * Ai[nn * ntau + tau] * Ai[mm * ntau + tau];",
     "tuple_weight(tau) * Ai[nn * ntau + tau] * Ai[nn * ntau + tau];",
     lambda: pairden.test_pair_density_matches_pairwise_formula_every_layer()),
]


@pytest.mark.parametrize("name,old,new,pin", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new, pin, tmp_path):
    src = open(oracle.SRC).read()
    olds, news = (old, new) if isinstance(old, tuple) else ((old,), (new,))
    for o, n_ in zip(olds, news):
        assert src.count(o) == 1, f"mutation site not found once: {o}"
        src = src.replace(o, n_)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    lib = oracle.compile_source(str(path), str(tmp_path / "libmutant.so"))
    with oracle.use_library(lib):
        with pytest.raises(AssertionError):
            pin()
    # the real oracle still passes the same pin
    pin()
