"""The FP8 kernels' division-free E4M3 quotient gives the codes of the IEEE
quotient: a strided run of the exhaustive check in tests/quotient_proof.c (the
full run, stride 1, covers all 5.3e8 bf16 (amax, y) pairs and is recorded in the
design notes)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_quotient_matches_ieee_division_in_e4m3(tmp_path):
    exe = os.path.join(tmp_path, "quotient_proof")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe,
                    os.path.join(HERE, "quotient_proof.c"), "-lm"], check=True)
    r = subprocess.run([exe, "97", "bf16", "near"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout
    assert "scale mismatches 0" in r.stdout and "pairs" in r.stdout
    assert r.stdout.strip().endswith("mismatches 0")


def test_quotient_matches_ieee_division_in_e4m3_fp16(tmp_path):
    """The same check over binary16 rows (the full run covers 5.0e8 pairs)."""
    exe = os.path.join(tmp_path, "quotient_proof")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe,
                    os.path.join(HERE, "quotient_proof.c"), "-lm"], check=True)
    r = subprocess.run([exe, "89", "fp16", "near"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout
    assert "scale mismatches 0" in r.stdout and "pairs" in r.stdout
    assert r.stdout.strip().endswith("mismatches 0")
