"""The oracle's pins are strong enough to catch plausible mistakes (no GPU).

Each case plants one mistake in a copy of an oracle module, on the CPU: a dropped term, a
wrong sign, an off-by-one bound, a transposed operand or index, a changed order.  A fresh
interpreter loads the mutated copy in place of the real module and runs that module's pin
file under pytest.  At least one pin must fail (pytest exit status 1).  The unmutated
oracle passes the same files in the normal suite.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Loads the oracle package, swaps one submodule for a mutated copy of its source, then runs
# one pin file.  Exit status 3: the text to replace is not found exactly once.
_BOOT = r"""
import os, sys, types
root, rel, modname, old, new, pins = sys.argv[1:7]
sys.path.insert(0, root)
import oracle
path = os.path.join(root, rel)
src = open(path).read()
if src.count(old) != 1:
    sys.exit(3)
mod = types.ModuleType(modname)
mod.__file__ = path
mod.__package__ = "oracle"
sys.modules[modname] = mod
exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)
setattr(oracle, modname.split(".")[1], mod)
import pytest
sys.exit(int(pytest.main([pins, "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"])))
"""

ATT = ("oracle/attention.py", "oracle.attention", "tests/test_oracle_attention.py")
REO = ("oracle/reorder.py", "oracle.reorder", "tests/test_oracle_reorder.py")
MSK = ("oracle/mask.py", "oracle.mask", "tests/test_oracle_mask.py")
CAL = ("oracle/calib.py", "oracle.calib", "tests/test_oracle_calib.py")

MUTANTS = {
    # block-masked attention
    "attn: scale dropped": (ATT, "s = sc * (q[b, h, rows]", "s = (q[b, h, rows]"),
    "attn: mask row read as a column": (ATT, "mask_row = masks[h if hm == H else 0, i]",
                                        "mask_row = masks[h if hm == H else 0, :, i]"),
    "attn: first head's mask for every head": (ATT, "mask_row = masks[h if hm == H else 0, i]",
                                               "mask_row = masks[0, i]"),
    "attn: first padding key attended": (ATT, "keys = keys[keys < n_valid]", "keys = keys[keys <= n_valid]"),
    "attn: LSE in base 2": (ATT, "lse[b, h, rows] = (m + np.log(l))", "lse[b, h, rows] = (m + np.log2(l))"),
    "attn: row sum not divided out": (ATT, "out[b, h, rows] = (e @ v[b, h, keys]) / l",
                                      "out[b, h, rows] = (e @ v[b, h, keys])"),
    "attn: K in place of V": (ATT, "out[b, h, rows] = (e @ v[b, h, keys])", "out[b, h, rows] = (e @ k[b, h, keys])"),
    "attn: max added instead of subtracted": (ATT, "e = np.exp(s - m)", "e = np.exp(s + m)"),
    "attn: empty row LSE 0": (ATT, "lse[b, h, rows] = -np.inf", "lse[b, h, rows] = 0.0"),
    "broadcast: LSE not copied": (ATT, "                    lse[b, h, i * block_size:(i + 1) * block_size] = lse[b, h, j * block_size:(j + 1) * block_size]\n",
                                  ""),
    "broadcast: rows copied from the block after the source": (
        ATT, "= out[b, h, j * block_size:(j + 1) * block_size]", "= out[b, h, (j + 1) % nb * block_size:((j + 1) % nb + 1) * block_size]"),
    "squad: global pass values are V": (ATT, "@ o_local[b, h, idx]", "@ v[b, h, idx]"),
    "squad: global pass over windows, not positions": (ATT, "idx = np.arange(p, n, window)",
                                                       "idx = np.arange(p * m, (p + 1) * m)"),
    "squad: local pass over positions": (ATT, "idx = np.arange(a * window, (a + 1) * window)",
                                         "idx = np.arange(a, n, m)"),
    # token reorder
    "reorder: w tiles before h tiles": (REO, "for h0 in range(0, H, th):\n            for w0 in range(0, W, tw):",
                                        "for w0 in range(0, W, tw):\n            for h0 in range(0, H, th):"),
    "reorder: last tile row dropped": (REO, "min(h0 + th, H)", "min(h0 + th, H - 1)"),
    "reorder: raster index transposed": (REO, "perm.append(t * H * W + h * W + w)", "perm.append(t * H * W + w * H + h)"),
    "reorder: padding rows not zeroed": (REO, "dst = np.zeros((src.shape[0], n_pad)", "dst = np.ones((src.shape[0], n_pad)"),
    "reorder: inverse gathers instead of scattering": (REO, "dst[:, perm[k]] = src[:, k]", "dst[:, k] = src[:, perm[k]]"),
    "reorder: tile depth ignored": (REO, "for t in range(t0, min(t0 + tt, T)):", "for t in range(t0, min(t0 + 1, T)):"),
    # masks and CSR
    "mask: window bounds strict": (MSK, "lo[j] <= hi[i] + radius and hi[j] >= lo[i] - radius",
                                   "lo[j] < hi[i] + radius and hi[j] > lo[i] - radius"),
    "mask: anchors rotate backwards": (MSK, "anchors.add((a * nb // num_anchors + step) % nb)",
                                       "anchors.add((a * nb // num_anchors - step) % nb)"),
    "mask: padding block takes its own unit": (MSK, "lo[i] = hi[i] = last_real_unit",
                                               "lo[i] = hi[i] = first // unit_tokens"),
    "mask: strided block in the previous group": (MSK, "m[i, (i + group) % nb] = True", "m[i, (i - group) % nb] = True"),
    "mask: CSR rows read transposed": (MSK, "js = [j for j in range(nb) if masks[h, i, j]]",
                                       "js = [j for j in range(nb) if masks[h, j, i]]"),
    "mask: LVSA window grows left first": (MSK, "if (turn_right and can_right) or not can_left:",
                                           "if (not turn_right and can_right) or not can_left:"),
    "mask: LVSA global frames rotate backwards": (MSK, "anchors = {(a * T // num_anchors + step) % T",
                                                  "anchors = {(a * T // num_anchors - step) % T"),
    "mask: two-stage groups shifted": (MSK, "if j // group == i // group:", "if (j + 1) // group == i // group:"),
    "mask: anchors spaced by nb // G": (MSK, "anchors.add((a * nb // num_anchors + step) % nb)",
                                        "anchors.add((a * (nb // num_anchors) + step) % nb)"),
    "mask: two-stage stride of one block": (MSK, "m[i, (i + group) % nb] = True", "m[i, (i + 1) % nb] = True"),
    "mask: LVSA global frames spaced by T // G": (MSK, "anchors = {(a * T // num_anchors + step) % T",
                                                  "anchors = {(a * (T // num_anchors) + step) % T"),
    "mask: LVSA block's last frame dropped": (MSK, "return range(first // frame_tokens, last // frame_tokens + 1)",
                                              "return range(first // frame_tokens, last // frame_tokens)"),
    "mask: LVSA budget one short": (MSK, "target = min(budget, T)", "target = min(budget, T) - 1"),
    # calibration
    "calib: energies not normalised": (CAL, "a = e / e.sum(axis=1, keepdims=True)", "a = e"),
    "calib: padding keys in the softmax": (CAL, "keys = k[b, h, :n_valid]", "keys = k[b, h, :]"),
    "calib: ascending energy order": (CAL, "key=lambda j: (-e[j], j)", "key=lambda j: (e[j], j)"),
    "calib: ties by descending index": (CAL, "key=lambda j: (-e[j], j)", "key=lambda j: (-e[j], -j)"),
    "calib: threshold strict": (CAL, "if prefix[kk] >= target:", "if prefix[kk] > target:"),
    "calib: padding query rows counted": (CAL, "r0, r1 = i * bs, min((i + 1) * bs, n_valid)", "r0, r1 = i * bs, (i + 1) * bs"),
    "calib: absolute threshold": (CAL, "target = float(eps) * prefix[n]", "target = float(eps)"),
    "calib: block mean instead of sum": (CAL, "energy[b, h, i, j] = a[:, c0:c1].sum()", "energy[b, h, i, j] = a[:, c0:c1].mean()"),
    "calib: one block too many": (CAL, "for j in order[:kcount]:", "for j in order[:kcount + 1]:"),
    "calib: agreement strict": (CAL, "return count >= float(rho) * float(p)", "return count > float(rho) * float(p)"),
}


# Not listed: mistakes that change nothing, so no pin can see them.  Examples are a
# partial last block taking the unit of its last padding token (that unit lies beyond
# every block's range anyway), and the energy softmax without the max subtraction (the
# normalisation cancels it).


def _run(case):
    (rel, modname, pins), old, new = MUTANTS[case]
    env = dict(os.environ, PYTHONPATH=ROOT, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-c", _BOOT, ROOT, rel, modname, old, new, pins], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return case, r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def outcomes():
    workers = max(1, min(8, os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        return {case: (rc, out) for case, rc, out in ex.map(_run, MUTANTS)}


@pytest.mark.parametrize("case", list(MUTANTS))
def test_planted_mistake_fails_a_pin(outcomes, case):
    rc, out = outcomes[case]
    assert rc != 3, f"{case}: the text to mutate is not in the oracle source (update the mutant)"
    assert rc == 1, f"{case}: no pin failed (pytest exit status {rc})\n{out}"
