"""Planted mistakes in the oracle, on the CPU.

Each mutant changes one step of an oracle function the way a plausible slip would: a dropped or
shifted factor, swapped operands, an off-by-one index, a reversed comparison, a missing
temperature.  A mutant is built by wrapping the real function (its inputs or outputs changed),
installed wherever the oracle and its pin tests refer to that function, and the pins of that
oracle function are run against it: at least one must fail.  Where a slip would sit in a step
that two oracle functions share (attention's flat and padded forms), both get it, so that the
pins that check one form against the other cannot be what catches it.
"""
import numpy as np
import pytest

import oracle.attention as O_attn
import oracle.calibration as O_cal
import oracle.draft as O_draft
import oracle.kv_commit as O_kv
import oracle.schedule as O_sched
from tests import test_oracle_accept as T_acc
from tests import test_oracle_attention as T_attn
from tests import test_oracle_calibration as T_cal
from tests import test_oracle_draft as T_draft
from tests import test_oracle_kv_commit as T_kv
from tests import test_oracle_schedule as T_sched


def _caught(monkeypatch, patches, pins):
    """True when some pin's assertion fails with the patched functions installed."""
    with monkeypatch.context() as m:
        for mod, name, fn in patches:
            m.setattr(mod, name, fn)
        for pin in pins:
            try:
                pin()
            except AssertionError:   # a pin's check; any other error is a broken mutant
                return True
    return False


def _everywhere(name, fn, modules):
    return [(mod, name, fn) for mod in modules if hasattr(mod, name)]


# ---------------------------------------------------------------- schedule
_survival, _order, _flatten = O_sched.survival_ref, O_sched.candidate_order, O_sched.flatten_ref

SCHEDULE_PINS = [
    T_sched.test_survival_is_product_of_conditionals,
    T_sched.test_candidate_order_tiebreak,
    T_sched.test_lag_two_rounds,
    T_sched.test_flat_table_takes_everything,
    T_sched.test_unit_cost_per_token_takes_nothing,
    lambda: T_sched.test_worked_scores_from_the_pages(0.1, 3),
    lambda: T_sched.test_worked_scores_from_the_pages(0.3, 2),
    *[(lambda s=s: T_sched.test_greedy_matches_bruteforce(s)) for s in range(4)],
    T_sched.test_invariants_and_markers,
    T_sched.test_flatten_layout,
]


def _survival_exclusive(conf):      # the product of the conditionals before position k
    S = _survival(conf)
    return np.concatenate([np.ones((S.shape[0], 1)), S[:, :-1]], axis=1)


def _survival_no_product(conf):     # the conditional itself, not the product
    return np.asarray(conf, dtype=np.float32).astype(np.float64)


def _order_ascending(S):
    order, s, r_of, k_of = _order(S)
    return np.lexsort((r_of, k_of, s)), s, r_of, k_of


def _order_r_before_k(S):
    order, s, r_of, k_of = _order(S)
    return np.lexsort((k_of, r_of, -s)), s, r_of, k_of


def _flatten_late(verify_len, kv_len):
    q_offsets, markers = _flatten(verify_len, kv_len)
    markers = markers.copy()
    markers[:, 1] += 1
    return q_offsets, markers


_schedule = O_sched.schedule_ref


def _objective_one_late(conf, kv_len, t_ms, T_cap):   # f(n) over the time of n + 1 tokens
    t = np.asarray(t_ms, dtype=np.float64)
    return _schedule(conf, kv_len, np.concatenate([t[1:], t[-1:]]), T_cap)


SCHEDULE_MUTANTS = {
    "survival without its first factor": ("survival_ref", _survival_exclusive),
    "survival without the product": ("survival_ref", _survival_no_product),
    "candidates by ascending survival": ("candidate_order", _order_ascending),
    "ties broken by request before position": ("candidate_order", _order_r_before_k),
    "confidences one round old": ("lagged_round", lambda i: max(i - 1, 0)),
    "markers one position late": ("flatten_ref", _flatten_late),
    "objective over the next batch size's time": ("schedule_ref", _objective_one_late),
}


@pytest.mark.parametrize("mutant", list(SCHEDULE_MUTANTS))
def test_schedule_pins_catch(monkeypatch, mutant):
    name, fn = SCHEDULE_MUTANTS[mutant]
    assert _caught(monkeypatch, _everywhere(name, fn, [O_sched, T_sched]), SCHEDULE_PINS), mutant


# ---------------------------------------------------------------- attention
_flat, _dense = O_attn.attn_ref_flat, O_attn.attn_ref_dense


def _both(transform):
    """The same slip in the flat and the padded form: transform(args dict) -> args dict."""
    def flat(q, k_new, v_new, kv_pages, block_table, kv_len, markers, q_offsets, scale,
             page_size, rows=None):
        a = transform(dict(q=q, k_new=k_new, v_new=v_new, kv_pages=kv_pages,
                           block_table=block_table, kv_len=kv_len, scale=scale))
        return _flat(a["q"], a["k_new"], a["v_new"], a["kv_pages"], a["block_table"],
                     a["kv_len"], markers, q_offsets, a["scale"], page_size, rows)

    def dense(q, k_new, v_new, kv_pages, block_table, kv_len, verify_len, scale, page_size):
        a = transform(dict(q=q, k_new=k_new, v_new=v_new, kv_pages=kv_pages,
                           block_table=block_table, kv_len=kv_len, scale=scale))
        return _dense(a["q"], a["k_new"], a["v_new"], a["kv_pages"], a["block_table"],
                      a["kv_len"], verify_len, a["scale"], page_size)
    return flat, dense


def _no_scale(a):
    return dict(a, scale=1.0)


def _swap_kv(a):
    pages = np.array(a["kv_pages"], copy=True)
    pages[:, [0, 1]] = pages[:, [1, 0]]
    return dict(a, k_new=a["v_new"], v_new=a["k_new"], kv_pages=pages)


def _logical_pages(a):
    bt = np.asarray(a["block_table"])
    ident = np.broadcast_to(np.arange(bt.shape[1]), bt.shape) + bt.shape[1] * np.arange(bt.shape[0])[:, None]
    return dict(a, block_table=np.where(bt >= 0, ident % np.asarray(a["kv_pages"]).shape[0], bt))


def _transposed_q(a):                 # query heads of a group read in reverse order
    q = np.asarray(a["q"])
    return dict(a, q=q[:, ::-1, :].copy())


def _one_key_short(a):
    return dict(a, kv_len=np.maximum(np.asarray(a["kv_len"]) - 1, 0))


ATTENTION_MUTANTS = {
    "scale dropped": _no_scale,
    "one cached key too few": _one_key_short,
    "keys and values swapped": _swap_kv,
    "block table ignored": _logical_pages,
    "query heads reversed": _transposed_q,
}

ATTENTION_PINS = [
    T_attn.test_dense_equals_sdpa_library_routine,
    T_attn.test_uniform_weights_closed_form,
    T_attn.test_single_visible_key_returns_its_value,
    T_attn.test_page_placement_does_not_matter,
    T_attn.test_dominant_key,
    T_attn.test_structured_keys_select_and_average_exactly,
    lambda: T_attn.test_flat_equals_dense(0),
]


@pytest.mark.parametrize("mutant", list(ATTENTION_MUTANTS))
def test_attention_pins_catch(monkeypatch, mutant):
    flat, dense = _both(ATTENTION_MUTANTS[mutant])
    patches = (_everywhere("attn_ref_flat", flat, [O_attn, T_attn]) +
               _everywhere("attn_ref_dense", dense, [O_attn, T_attn]))
    assert _caught(monkeypatch, patches, ATTENTION_PINS), mutant


# ---------------------------------------------------------------- acceptance
_accept = T_acc.accept_ref


def _accept_with(transform):
    def fn(target_logits, draft_logits, draft_tokens, verify_len, q_offsets, u_acc, u_res,
           temperature, chunk_bytes=1 << 28):
        a = transform(dict(target_logits=target_logits, draft_logits=draft_logits,
                           u_acc=u_acc, u_res=u_res, temperature=temperature))
        return _accept(a["target_logits"], a["draft_logits"], draft_tokens, verify_len,
                       q_offsets, a["u_acc"], a["u_res"], a["temperature"], chunk_bytes)
    return fn


def _u_reversed(a):
    return dict(a, u_acc=(1.0 - np.asarray(a["u_acc"], np.float64)).astype(np.float32))


def _no_temperature(a):
    return dict(a, temperature=1.0 if a["temperature"] > 0 else a["temperature"])


def _draft_neighbour(a):
    return dict(a, draft_logits=np.roll(np.asarray(a["draft_logits"]), 1, axis=1))


def _residual_reuses_acceptance_uniform(a):
    ur = np.array(a["u_res"], copy=True)
    ur[:, :ur.shape[1] - 1] = a["u_acc"]
    return dict(a, u_res=ur)


ACCEPT_MUTANTS = {
    "uniform compared the wrong way": _u_reversed,
    "temperature ignored": _no_temperature,
    "draft row of the neighbouring position": _draft_neighbour,
    "residual drawn with the acceptance uniform": _residual_reuses_acceptance_uniform,
}

ACCEPT_PINS = [                       # cheapest first: the run stops at the first failure
    T_acc.test_deterministic_decisions,
    T_acc.test_greedy_matches_argmax_loop,
    T_acc.test_invariants_random,
    T_acc.test_flags_mark_threshold_cases,
    T_acc.test_zero_uniform_picks_first_positive_mass,
    T_acc.test_empty_residual_draws_from_target,
    T_acc.test_equal_distributions_accept_everything,
    T_acc.test_first_token_follows_the_tempered_target,
    T_acc.test_three_token_joint_position_dependent,
    T_acc.test_first_token_v32_position_dependent,
]


@pytest.mark.parametrize("mutant", list(ACCEPT_MUTANTS))
def test_accept_pins_catch(monkeypatch, mutant):
    fn = _accept_with(ACCEPT_MUTANTS[mutant])
    assert _caught(monkeypatch, [(T_acc, "accept_ref", fn)], ACCEPT_PINS), mutant


# ---------------------------------------------------------------- KV commit
_commit = O_kv.kv_commit_ref


def _commit_with(da=0, swap=False, late=0):
    def fn(k_new, v_new, caches, block_table, kv_len, q_offsets, accepted_len, K, T_cap):
        a = np.asarray(accepted_len) + da
        if swap:
            k_new, v_new = v_new, k_new
        return _commit(k_new, v_new, caches, block_table, np.asarray(kv_len) + late, q_offsets,
                       a, K, T_cap)
    return fn


COMMIT_MUTANTS = {
    "one token too few": _commit_with(da=-1),
    "one token too many": _commit_with(da=+1),
    "keys and values swapped": _commit_with(swap=True),
    "written one position late": _commit_with(late=1),
}

COMMIT_PINS = [
    lambda: T_kv.test_attention_over_committed_cache_equals_attention_over_kept_verify_rows(0),
    T_kv.test_only_the_kept_slots_change_and_rejected_rows_never_appear,
    T_kv.test_each_layer_gets_its_own_rows,
    T_kv.test_zero_accepted_commits_only_the_first_verify_token,
]


@pytest.mark.parametrize("mutant", list(COMMIT_MUTANTS))
def test_commit_pins_catch(monkeypatch, mutant):
    fn = COMMIT_MUTANTS[mutant]
    assert _caught(monkeypatch, _everywhere("kv_commit_ref", fn, [O_kv, T_kv]), COMMIT_PINS), mutant


# ---------------------------------------------------------------- calibration
_calibrate, _fit, _outcomes = O_cal.calibrate_ref, O_cal.fit_temperature_ref, O_cal.outcomes_from_accept

CALIBRATION_MUTANTS = {
    "logit multiplied by the temperature": ("calibrate_ref", lambda l, t: _calibrate(l, 1.0 / np.asarray(t, np.float64))),
    "fit returns 1 / temperature": ("fit_temperature_ref", lambda *a: 1.0 / _fit(*a)),
    "outcomes one position late": ("outcomes_from_accept", lambda *a: np.roll(_outcomes(*a), 1, axis=1)),
    "logit sign flipped": ("calibrate_ref", lambda l, t: _calibrate(-np.asarray(l), t)),
}

CALIBRATION_PINS = [
    T_cal.test_tau_one_is_the_logistic_function_and_symmetric,
    T_cal.test_outcomes_follow_the_accepted_prefix,
    T_cal.test_fit_is_the_likelihood_minimiser_of_a_library_routine,
    T_cal.test_planted_temperature_is_recovered,
]


@pytest.mark.parametrize("mutant", list(CALIBRATION_MUTANTS))
def test_calibration_pins_catch(monkeypatch, mutant):
    name, fn = CALIBRATION_MUTANTS[mutant]
    assert _caught(monkeypatch, _everywhere(name, fn, [O_cal, T_cal]), CALIBRATION_PINS), mutant


# ---------------------------------------------------------------- Markov-head draft
_draft = O_draft.markov_draft_ref

DRAFT_MUTANTS = {
    "temperature ignored": lambda B, E, U, x0, tau, round_idx, seed=0: _draft(
        B, E, U, x0, 1.0 if tau > 0 else tau, round_idx, seed),
    "previous token ignored": lambda B, E, U, x0, tau, round_idx, seed=0: _draft(
        B, E, U, np.zeros_like(np.asarray(x0)), tau, round_idx, seed),
    "transition transposed": lambda B, E, U, x0, tau, round_idx, seed=0: _draft(
        B, np.asarray(U).T, np.asarray(E).T, x0, tau, round_idx, seed),
    "previous token off by one": lambda B, E, U, x0, tau, round_idx, seed=0: _draft(
        B, E, U, (np.asarray(x0) + 1) % np.asarray(B).shape[-1], tau, round_idx, seed),
}

DRAFT_PINS = [
    T_draft.test_forced_transition_walks_the_vocabulary,
    T_draft.test_greedy_without_transition_is_the_library_argmax,
    T_draft.test_sampled_token_follows_softmax_of_the_tempered_logits,
]


@pytest.mark.parametrize("mutant", list(DRAFT_MUTANTS))
def test_draft_pins_catch(monkeypatch, mutant):
    fn = DRAFT_MUTANTS[mutant]
    assert _caught(monkeypatch, _everywhere("markov_draft_ref", fn, [O_draft, T_draft]),
                   DRAFT_PINS), mutant


def test_the_pins_pass_on_the_oracle_as_it_is(monkeypatch):
    """The same runs with nothing planted: every pin above passes, so a catch is the mutant's."""
    for pins in (SCHEDULE_PINS, ATTENTION_PINS, COMMIT_PINS, CALIBRATION_PINS, DRAFT_PINS,
                 ACCEPT_PINS[:7]):
        assert not _caught(monkeypatch, [], pins)
