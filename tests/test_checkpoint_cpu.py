"""Codebook checkpoints (decode_attention_commvq_b200/checkpoint.py) on the CPU: the file format
round-trips and rejects damaged or foreign files, and a fit interrupted at any EM step and
resumed from its checkpoint ends with the uninterrupted fit's codebook bit for bit. The fit's two
steps come from the oracle here (the GPU fit plugs in the library's calls instead)."""
import numpy as np
import pytest

from decode_attention_commvq_b200 import checkpoint as C
from decode_attention_commvq_b200 import synth
from oracle import oracle as O


def _state(**kw):
    base = dict(d=16, g=8, R=2, n_codes=4, rounds_done=1, iters_done=2, iters=3, seed=7)
    base.update(kw)
    return C.FitState(**base)


def test_round_trip(tmp_path):
    p = str(tmp_path / "cb.bin")
    cb = np.random.default_rng(1).standard_normal((2, 2, 4, 8)).astype(np.float32)
    st = _state()
    C.save(p, cb, st)
    cb2, st2 = C.load(p)
    assert st2 == st and np.array_equal(cb2.view(np.uint32), cb.view(np.uint32))
    assert (tmp_path / "cb.bin").stat().st_size == 64 + cb.nbytes


def test_rejects_damaged_and_foreign_files(tmp_path):
    p = str(tmp_path / "cb.bin")
    cb = np.zeros((2, 2, 4, 8), dtype=np.float32)
    C.save(p, cb, _state())
    raw = open(p, "rb").read()
    for bad, what in ((raw[:-4], "data bytes"), (b"NOTACBKP" + raw[8:], "magic"), (raw[:30], "too short"),
                      (raw[:8] + (2).to_bytes(4, "little") + raw[12:], "version")):
        open(p, "wb").write(bad)
        with pytest.raises(ValueError, match=what):
            C.load(p)
    with pytest.raises(ValueError, match="shape"):
        C.save(p, np.zeros((1, 2, 4, 8), np.float32), _state())


def _oracle_steps(w):
    def em_step(res, cb_r):
        return O.em_step(res, cb_r)[0]

    def advance(res, cb_r):
        return O.encode(res, cb_r[None], want_residual=True)[2]

    def seed_round(res, r):
        return O.forgy_init(res, synth.forgy_indices(w, True, r, res.shape[0]), w.g)

    return C.FitSteps(em_step=em_step, advance=advance, seed_round=seed_round,
                      to_numpy=lambda a: np.asarray(a, dtype=np.float32), from_numpy=lambda a: a.copy())


class _Stop(Exception):
    pass


@pytest.mark.parametrize("stop_after", [0, 1, 2, 3, 4])
def test_interrupted_fit_resumes_to_the_same_codebook(tmp_path, stop_after):
    """R = 2 rounds x 3 EM steps: interrupted after EM step `stop_after` (0-2 round 0, 3-4 round 1;
    step 2 ends round 0), then resumed from the file."""
    w = synth.WORKLOADS[1].with_(em_rows=300, n_codes=16, R=2)
    rows = synth.fit_rows(w, True)
    steps = _oracle_steps(w)
    full = C.resumable_fit(rows, 2, 8, 16, 3, steps)
    ref, _ = O.fit_codebook(rows, 2, 8, 16, 3, lambda r, N: synth.forgy_indices(w, True, r, N))
    assert np.array_equal(np.stack(full).view(np.uint32), ref.view(np.uint32))   # the driver is the fit
    p = str(tmp_path / "fit.bin")
    count = [0]

    def stop(r, it):
        if count[0] == stop_after:
            raise _Stop()
        count[0] += 1

    with pytest.raises(_Stop):
        C.resumable_fit(rows, 2, 8, 16, 3, steps, path=p, seed=5, on_step=stop)
    _, st = C.load(p)
    assert st.rounds_done * 3 + st.iters_done == stop_after + 1
    resumed = C.resumable_fit(rows, 2, 8, 16, 3, steps, path=p, seed=5)
    assert np.array_equal(np.stack(resumed).view(np.uint32), np.stack(full).view(np.uint32))
    _, st = C.load(p)
    assert st.finished and st.rounds_done == 2
    with pytest.raises(ValueError, match="another fit"):
        C.resumable_fit(rows, 2, 8, 16, 3, steps, path=p, seed=6)
