"""The diagonal-only ablation on the synthetic Llama-layer recipe, in the oracle.

The KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
§数学主线二) builds the pair objective with a coupling term between the two Keys;
dropping it (g12 = 0) gives the per-key weighting it contrasts with. This measures
what the coupling buys on this repository's synthetic inputs: how much the diagonal
merged Key raises the coupled objective, how often the two forms pick different
pairs, and the decode error of each compressed cache against attention over the
uncompressed one. The numbers are printed (run with -s); the assertions are the
ones that hold by construction.
"""

import numpy as np
import pytest

import oracle
from asymmetric_kv_merging_b200 import inputs


def _layer(T=2048, H_kv=2, seed_layer=0, q_scale=1.0):
    w = inputs.small_workload(inputs.workload(1), H_kv=H_kv, H_q=4 * H_kv, T=T, n_decode=8)
    li = inputs.make_layer(w, seed_layer, q_scale=q_scale)
    return w, li


def _full_objective(w, n11, n12, n22, dsq):
    # the coupled objective at k = k_a + w (k_b - k_a), written out
    return dsq * (n11 * w * w - 2.0 * n12 * w * (w - 1.0) + n22 * (w - 1.0) ** 2)


# q_scale 1: the recipe as drawn (window-mean attention ~ 1/T per row, so the coupling
# N12 ~ a_a a_b is ~1/T of the self terms); 6: peaked attention, where it is not
@pytest.mark.parametrize("q_scale", [1.0, 6.0])
def test_diagonal_form_costs_objective_and_changes_selection(q_scale):
    w, li = _layer(q_scale=q_scale)
    K = li.K.double().numpy()
    V = li.V.double().numpy()
    lens = li.lens.numpy()
    Q = li.Q_win.double().numpy()
    G = w.H_q // w.H_kv
    excess, differ, total = [], 0, 0
    for h in range(w.H_kv):
        L = int(lens[0, h])
        args = (K[0, h], V[0, h], None, L, w.sink, w.W, Q[0, h * G:(h + 1) * G], w.W)
        full = oracle.score_head(*args)
        diag = oracle.score_head(*args, form="diagonal")
        a = w.sink + 2 * np.arange(full.score.shape[0])
        dsq = np.sum((K[0, h, a + 1] - K[0, h, a]) ** 2, axis=1)
        f_full = _full_objective(full.w_b, full.n11, full.n12, full.n22, dsq)
        f_diag = _full_objective(diag.w_b, full.n11, full.n12, full.n22, dsq)
        ok = ~full.degenerate & ~diag.degenerate
        assert np.all(f_full[ok] <= f_diag[ok] + 1e-9 * np.abs(f_diag[ok]) + 1e-300)
        pos = ok & (f_full > 0)
        excess.append(f_diag[pos] / f_full[pos] - 1.0)
        # the pairs a merge of a quarter of them would pick
        R = full.score.shape[0] // 4
        differ += int(np.sum(oracle.select_pairs(full.score, R) != oracle.select_pairs(diag.score, R)))
        total += 2 * R
    ex = np.concatenate(excess)
    print(f"\nq_scale {q_scale}: diagonal form: coupled objective raised by {100 * np.median(ex):.3g}% (median), "
          f"{100 * np.mean(ex):.3g}% (mean) over {ex.size} pairs; "
          f"selections of a quarter of the pairs differ in {100 * differ / total:.3g}% of picks")
    assert ex.size > 0 and np.all(ex >= -1e-9)


@pytest.mark.parametrize("q_scale", [1.0, 6.0])
def test_decode_error_of_each_form_against_the_uncompressed_cache(q_scale):
    w, li = _layer(q_scale=q_scale)
    B, H = 1, w.H_kv
    lens = li.lens.numpy().astype(np.int64)
    Q = li.Q_win.double().numpy()
    q = li.q_dec.double().numpy()                        # [n_decode, B, H_q, d]
    base = oracle.cache_from_arrays(li.K.double().numpy(), li.V.double().numpy(), lens)
    ref = np.stack([oracle.decode_step(base, q[s])[0] for s in range(q.shape[0])])
    target = lens // 2
    errs = {}
    for form in oracle.FORMS:
        cache, rounds = oracle.compress(base, Q, w.W, np.full((B, H), w.sink), w.W, target,
                                        form=form)
        assert np.all(cache.lengths() == target)
        out = np.stack([oracle.decode_step(cache, q[s])[0] for s in range(q.shape[0])])
        errs[form] = float(np.linalg.norm(out - ref) / np.linalg.norm(ref))
    print(f"\nq_scale {q_scale}: decode relative error after 2x compression: full form {errs['full']:.4g}, "
          f"diagonal form {errs['diagonal']:.4g}")
    assert all(np.isfinite(v) for v in errs.values())
