"""Mutation check of the oracle pins (CPU only).

Each case plants one plausible slip in a private copy of the oracle (a dropped scale, an off-by-one or
mis-aligned mask, a wrong log base, a missing normalisation, a sign flip, a broken merge or gradient
term) and runs the oracle pins against that copy: every mutant must make them fail, while the
unmodified copy must pass.  The repository's own files are never edited.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (file under oracle/, text to replace, replacement)
MUTANTS = {
    "drop_scale": ("attention.py", "s = scale * (q @ k.T)", "s = (q @ k.T)"),
    "causal_off_by_one": ("attention.py", "vis &= (j <= i + (nk - nq)) | (j < prefix)",
                          "vis &= (j < i + (nk - nq)) | (j < prefix)"),
    "causal_top_left": ("attention.py", "vis &= (j <= i + (nk - nq)) | (j < prefix)",
                        "vis &= (j <= i) | (j < prefix)"),
    "prefix_off_by_one": ("attention.py", "vis &= (j <= i + (nk - nq)) | (j < prefix)",
                          "vis &= (j <= i + (nk - nq)) | (j <= prefix)"),
    "key_length_off_by_one": ("attention.py", "vis &= j < k_valid", "vis &= j <= k_valid"),
    "lse_log2": ("attention.py", "lse[live] = m + np.log(l)", "lse[live] = m + np.log2(l)"),
    "lse_without_max": ("attention.py", "lse[live] = m + np.log(l)", "lse[live] = np.log(l)"),
    "no_normalisation": ("attention.py", "o[live] = (p @ v) / l[:, None]", "o[live] = (p @ v)"),
    "exp_sign": ("attention.py", "p = np.exp(sl - m[:, None])", "p = np.exp(m[:, None] - sl)"),
    "shard_offset_sign": ("attention.py", "min(max(int(L) - key_offset, 0), nk)",
                          "min(max(int(L) + key_offset, 0), nk)"),
    "tiled_no_rescale": ("online.py", "acc = alpha[:, None] * acc + p @ vj", "acc = acc + p @ vj"),
    "merge_drops_weight": ("online.py", "return m, np.concatenate([e1 * f1, e2 * f2]), e1 * l1 + e2 * l2",
                           "return m, np.concatenate([f1, e2 * f2]), l1 + e2 * l2"),
    "combine_old_weight": ("online.py", "acc = e_old * acc + e_s * o_s", "acc = acc + e_s * o_s"),
    "bwd_drop_row_term": ("backward.py", "ds = p * (dp - drow[:, None])", "ds = p * dp"),
    "bwd_dq_no_scale": ("backward.py", "dq = scale * (ds @ k)", "dq = ds @ k"),
    "bwd_dk_transposed": ("backward.py", "dk = scale * (ds.T @ q)", "dk = scale * (ds @ q)[: q.shape[0]]"),
    "bwd_prefix_ignored": ("backward.py", "q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale, causal, prefix)",
                           "q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale, causal, 0)"),
    "bwd_varlen_prefix_ignored": ("backward.py", "do[s0:s1, h], scale, causal, prefix)",
                                  "do[s0:s1, h], scale, causal, 0)"),
    "bwd_rows_drop_row_term": ("backward.py", "dsc = pc * (do[a:e] @ v[cols].T - drow[:, None])",
                               "dsc = pc * (do[a:e] @ v[cols].T)"),
    "bwd_rows_chunk_offset": ("attention.py", "i = np.arange(row_lo, row_hi)[:, None]",
                              "i = np.arange(0, row_hi - row_lo)[:, None]"),
    "bwd_rows_dv_uses_ds": ("backward.py", "dv += pc.T @ do[a:e]", "dv += dsc.T @ do[a:e]"),
    "paged_table_ignored": ("attention.py", "page = int(block_table[b][i])", "page = i"),
    "paged_partial_page_dropped": ("attention.py", "for i in range(-(-L // ps)):", "for i in range(L // ps):"),
    "paged_row_in_page": ("attention.py", "k_g[b, i * ps:(i + 1) * ps] = k_pages[page]",
                          "k_g[b, i * ps:(i + 1) * ps] = k_pages[page][::-1]"),
    "gqa_head_modulo": ("attention.py", "k_cache[b, :L, h // G, :], v_cache[b, :L, h // G, :]",
                        "k_cache[b, :L, h % Hkv, :], v_cache[b, :L, h % Hkv, :]"),
    "varlen_key_offset": ("attention.py", "k[s0:s1, h, :]", "k[:s1 - s0, h, :]"),
    "padded_mask_on_queries": ("attention.py", "s = np.where(kv[None, :], s, -np.inf)",
                               "s = np.where(kv[:, None], s, -np.inf)"),
    "split_floor": ("online.py", "per = -(-nk // num_splits)", "per = max(1, nk // num_splits)"),
    "split_lse_without_max": ("online.py", "lse[s] = m + math.log(l)", "lse[s] = math.log(l)"),
    "tiled_l_not_rescaled": ("online.py", "l = alpha * l + p.sum(axis=1)", "l = l + p.sum(axis=1)"),
    "tiled_causal_top_left": ("online.py", "cols[None, :] <= rows[:, None] + (nk - nq)", "cols[None, :] <= rows[:, None]"),
    "bwd_dv_untransposed": ("backward.py", "dv = p.T @ do",
                            "dv = (p @ do)[: v.shape[0]] if p.shape[0] >= v.shape[0] else p.T @ do"),
    "bwd_varlen_key_offset": ("backward.py", "q[s0:s1, h], k[s0:s1, h], v[s0:s1, h]",
                              "q[s0:s1, h], k[:s1 - s0, h], v[s0:s1, h]"),
}


def _tree(dst):
    """A private copy of what the pins need: the oracle, the input generator and the pins."""
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copy(os.path.join(ROOT, "seeded_inputs.py"), dst)
    shutil.copy(os.path.join(ROOT, "pytest.ini"), dst)
    os.makedirs(os.path.join(dst, "tests"))
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))


def _run_pins(dst):
    env = dict(os.environ, PYTHONPATH=dst, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "tests/test_oracle_pins.py"], cwd=dst,
                       env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout.strip().splitlines() or [""])[-1]


def _case(base, name):
    dst = os.path.join(base, name)
    _tree(dst)
    if name != "unmodified":
        fname, old, new = MUTANTS[name]
        path = os.path.join(dst, "oracle", fname)
        src = open(path).read()
        assert src.count(old) == 1, f"{name}: anchor not found once in oracle/{fname}"
        open(path, "w").write(src.replace(old, new))
    return name, _run_pins(dst)


@pytest.mark.slow
def test_every_mutant_fails_the_pins(tmp_path):
    names = ["unmodified"] + list(MUTANTS)
    with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
        results = dict(ex.map(lambda n: _case(str(tmp_path), n), names))
    rc, last = results.pop("unmodified")
    assert rc == 0, f"the unmodified copy must pass: {last}"
    survivors = {n: last for n, (rc, last) in results.items() if rc == 0}
    assert not survivors, f"mutants not caught by the pins: {survivors}"
