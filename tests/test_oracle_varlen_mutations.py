"""The packed-batch pins catch planted mistakes in the oracle's Python slicing.

oracle.fwd_varlen and oracle.bwd_varlen cut a packed batch into sequences and
hand each to the pinned C oracle; their own arithmetic is the slicing and the
placement of the results.  Each case copies the oracle package into a
temporary directory, plants one plausible mistake in oracle.py (keys cut with
the query bounds, a mask flag, window or ALiBi slopes not passed on, the last
key dropped, LSE or a gradient put in the wrong rows, the wrong upstream
gradient rows), and runs the packed-batch pins of test_oracle_varlen.py
against the copy in a child process, with the real C library.  The pins must
fail for every mutant.  Nothing here touches the real oracle package.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "oracle")

FWD_CALL = ("        ob, lb = fwd(_heads(q[q0:q1]), _heads(k[k0:k1]), _heads(v[k0:k1]), scale, flags, nthreads=nthreads,\n"
            "                     window=window, slopes=slopes)\n")
BWD_CALL = ("        ob, lb, dqb, dkb, dvb = bwd_full(_heads(q[q0:q1]), _heads(k[k0:k1]), _heads(v[k0:k1]),\n"
            "                                         _heads(dout[q0:q1]), scale, flags, nthreads=nthreads, window=window,\n"
            "                                         slopes=slopes)\n")

MUTANTS = {
    "fwd_keys_cut_with_query_bounds": (FWD_CALL, FWD_CALL.replace("k[k0:k1]", "k[q0:q1]").replace("v[k0:k1]", "v[q0:q1]")),
    "fwd_mask_flags_not_passed": (FWD_CALL, FWD_CALL.replace("scale, flags,", "scale, 0,")),
    "fwd_window_not_passed": (FWD_CALL, FWD_CALL.replace("window=window,", "window=None,")),
    "fwd_slopes_not_passed": (FWD_CALL, FWD_CALL.replace("slopes=slopes)", "slopes=None)")),
    "fwd_last_key_dropped": (FWD_CALL, FWD_CALL.replace("k[k0:k1]", "k[k0:max(k0 + 1, k1 - 1)]")
                             .replace("v[k0:k1]", "v[k0:max(k0 + 1, k1 - 1)]")),
    "fwd_lse_rows_reversed": ("        lse[:, q0:q1] = lb\n    return o, lse\n",
                              "        lse[:, q0:q1] = lb[:, ::-1]\n    return o, lse\n"),
    "bwd_mask_flags_not_passed": (BWD_CALL, BWD_CALL.replace("scale, flags,", "scale, 0,")),
    "bwd_window_not_passed": (BWD_CALL, BWD_CALL.replace("window=window,", "window=None,")),
    "bwd_upstream_gradient_of_other_rows": (BWD_CALL, BWD_CALL.replace("dout[q0:q1]", "dout[::-1][q0:q1]")),
    "bwd_dv_takes_dk": ("        dv[k0:k1] = np.transpose(dvb, (1, 0, 2))\n",
                        "        dv[k0:k1] = np.transpose(dkb, (1, 0, 2))\n"),
    "bwd_dq_rows_reversed": ("        dq[q0:q1] = np.transpose(dqb, (1, 0, 2))\n",
                             "        dq[q0:q1] = np.transpose(dqb, (1, 0, 2))[::-1]\n"),
}


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    """Runs the packed-batch pins against every mutant at once (child
    processes); returns {name: (returncode, tail of the output)}."""
    import oracle
    lib = oracle.build()                     # the real C library, unchanged
    src = open(os.path.join(PKG, "oracle.py")).read()
    test_src = os.path.join(ROOT, "tests", "test_oracle_varlen.py")
    procs = {}
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, f"mutation anchor not found once for {name}"
        assert new != old, name
        d = tmp_path_factory.mktemp(name)
        pkg = d / "oracle"
        pkg.mkdir()
        shutil.copy(os.path.join(PKG, "__init__.py"), pkg / "__init__.py")
        (pkg / "oracle.py").write_text(src.replace(old, new))
        shutil.copy(test_src, d / "test_oracle_varlen.py")
        env = dict(os.environ, ORACLE_LIB=lib, ORACLE_THREADS="2", PYTHONPATH=str(d))
        procs[name] = subprocess.Popen([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                                        "--rootdir", str(d), str(d / "test_oracle_varlen.py")],
                                       cwd=str(d), env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                       text=True)
    out = {}
    for name, pr in procs.items():
        text, _ = pr.communicate(timeout=600)
        out[name] = (pr.returncode, text[-2000:])
    return out


def test_unmutated_copy_passes(tmp_path):
    """The harness itself: the same copy without a mutation passes the pins."""
    import oracle
    lib = oracle.build()
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    shutil.copy(os.path.join(PKG, "__init__.py"), pkg / "__init__.py")
    shutil.copy(os.path.join(PKG, "oracle.py"), pkg / "oracle.py")
    shutil.copy(os.path.join(ROOT, "tests", "test_oracle_varlen.py"), tmp_path / "test_oracle_varlen.py")
    env = dict(os.environ, ORACLE_LIB=lib, ORACLE_THREADS="2", PYTHONPATH=str(tmp_path))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "--rootdir",
                        str(tmp_path), str(tmp_path / "test_oracle_varlen.py")],
                       cwd=str(tmp_path), env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_packed_pins_catch_mutant(name, mutant_runs):
    rc, tail = mutant_runs[name]
    assert rc != 0, f"mutant {name} survived the packed-batch pins:\n{tail}"
