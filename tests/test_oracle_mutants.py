"""Every plausible mistake in ``oracle_mutants.MUTANTS``, planted in the CPU
oracle one at a time in a child process, makes the oracle's pins fail.

This is the evidence that the pins pin the oracle to something other than
itself: a dropped term, a flipped sign, a transposed operand, a wrong index
or a wrong rounding anywhere in it changes a result that a hand-worked
example, a closed form, a brute-force solve or an invariant fixes."""
import concurrent.futures as cf
import os
import subprocess
import sys

import oracle_mutants

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PINS = [os.path.join(HERE, "test_oracle_pins.py"), os.path.join(HERE, "test_oracle_checkpoint.py")]


def _run(name):
    env = dict(os.environ, GPTQ_ORACLE_MUTANT=name, OMP_NUM_THREADS="1",
               OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-400:] + r.stderr[-400:]


def test_every_planted_mistake_fails_a_pin():
    workers = max(1, min(8, os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(_run, sorted(oracle_mutants.MUTANTS)))
    # exit status 1: tests ran and at least one failed (2-5 would be an
    # interrupted or broken run, not a caught mistake)
    survivors = [(n, rc, tail) for n, rc, tail in results if rc != 1]
    assert not survivors, survivors


def test_mutant_texts_occur_in_the_oracle():
    """Each substitution names text that is really in the function it
    mutates (a mutant that does not apply would prove nothing)."""
    from oracle import gptq_oracle as M
    for name, edits in oracle_mutants.MUTANTS.items():
        for fname, old, _ in edits:
            assert hasattr(M, fname), (name, fname)
            oracle_mutants._rewrite(M, fname, [(old, old)])
