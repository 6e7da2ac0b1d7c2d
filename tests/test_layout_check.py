"""The host-side dispatch-layout checker (moe_check_dispatch_host, no GPU): it accepts the
oracle's layouts ("Mixture-of-Experts : routage et capacité", "L'idée — Capacité" and
"Support visuel — Capacité") and names the first broken invariant of a corrupted one."""
import numpy as np
import pytest

import oracle as O
from mixture_experts_layer_50_b200 import _native as nat


def _layout(seed, N=200, E=8, k=2, cf=1):
    rng = np.random.default_rng(seed)
    z = rng.normal(0, 1, (N, E)).astype(np.float32)
    z[:, 0] += 1.5                                  # a hot expert: capacity drops some
    ids, _ = O.route(z, k)
    C = O.capacity(N, k, E, cf)
    d = O.dispatch(ids, E, C)
    return dict(ids=ids, drop_mask=d["drop_mask"], counts=d["counts"], demand=d["demand"],
                offsets=d["offsets"], slot_row=d["slot_row"], row_token=d["row_token"]), C


def _check(lay, C, N=200, E=8, k=2):
    return nat.moe_check_dispatch_host(N, k, E, C, **lay)


@pytest.mark.parametrize("seed,cf", [(0, 1), (1, 1.25), (2, None), (3, 0.5)])
def test_oracle_layouts_pass(seed, cf):
    lay, C = _layout(seed, cf=cf)
    assert _check(lay, C) == (nat.MOE_OK, "")


def _corrupt(fn):
    lay, C = _layout(7)
    lay = {n: np.array(v) for n, v in lay.items()}
    C = fn(lay, C)
    return _check(lay, C)


def _kept_rows(lay, e):
    return lay["slot_row"][(lay["ids"] == e) & (lay["drop_mask"] == 0)]


def test_each_broken_invariant_is_named():
    bad = nat.MOE_ERR_INVALID_INPUT

    def swap_two_rows_of_expert_0(lay, C):
        t = np.argwhere((lay["ids"] == 0) & (lay["drop_mask"] == 0))[:2]
        (a, ja), (b, jb) = t
        lay["slot_row"][a, ja], lay["slot_row"][b, jb] = lay["slot_row"][b, jb], lay["slot_row"][a, ja]
        lay["row_token"] = None
        return C

    cases = {
        "token order": swap_two_rows_of_expert_0,
        "out of range": lambda lay, C: (lay["ids"].__setitem__((5, 0), 99), C)[1],
        "twice": lambda lay, C: (lay["ids"].__setitem__((5, 1), lay["ids"][5, 0]), C)[1],
        "offsets step": lambda lay, C: (lay["offsets"].__setitem__(3, lay["offsets"][3] + 1), C)[1],
        "capacity": lambda lay, C: C - 1,
        "dropped but has row": lambda lay, C: (lay["slot_row"].__setitem__(
            tuple(np.argwhere(lay["drop_mask"] == 1)[0]), 0), C)[1],
        "maps to token": lambda lay, C: (lay["row_token"].__setitem__(0, lay["row_token"][0] + 1), C)[1],
    }
    for want, fn in cases.items():
        st, msg = _corrupt(fn)
        assert st == bad and want in msg, (want, msg)


def test_a_kept_token_after_a_dropped_one_is_caught():
    """Move expert 0's cut: keep its first dropped token and drop its last kept one (counts
    and offsets unchanged), which breaks the token-order capacity rule."""
    lay, C = _layout(11)
    ids, drop, slot = lay["ids"], lay["drop_mask"].copy(), lay["slot_row"].copy()
    kept = np.argwhere((ids == 0) & (drop == 0))
    dropped = np.argwhere((ids == 0) & (drop == 1))
    assert len(dropped) > 0
    (tk, jk), (td, jd) = kept[-1], dropped[0]
    row = slot[tk, jk]
    drop[tk, jk], slot[tk, jk] = 1, -1
    drop[td, jd], slot[td, jd] = 0, row
    lay.update(drop_mask=drop, slot_row=slot, row_token=None)
    st, msg = _check(lay, C)
    assert st == nat.MOE_ERR_INVALID_INPUT and "after dropping" in msg, msg


def test_counts_beyond_demand_and_bad_arguments():
    lay, C = _layout(12)
    lay["demand"] = np.array(lay["demand"])
    lay["demand"][2] = lay["counts"][2] - 1
    st, msg = _check(lay, C)
    assert st == nat.MOE_ERR_INVALID_INPUT and "demand" in msg
    st, _ = nat.moe_check_dispatch_host(-1, 2, 8, 0, ids=lay["ids"], drop_mask=lay["drop_mask"],
                                        counts=lay["counts"], offsets=lay["offsets"],
                                        slot_row=lay["slot_row"])
    assert st == nat.MOE_ERR_INVALID_ARG
