"""Plant plausible mistakes in a copy of the oracle and check that the CPU pins catch each.

    python tests/mutation_check.py

Each mutation is one textual edit of ``oracle/block.py`` (a dropped term, a wrong sign,
index, order, constant or exponent) applied to a copy of the oracle, tests and input
generators in a temporary directory; the pin tests (``test_oracle.py`` and
``test_tp_host.py``) then run there and must fail. The repository itself is never
modified. Exit status 1 if any mutation survives.
"""

import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "rotate_half sign": ("np.concatenate([-x[..., half:], x[..., :half]]",
                         "np.concatenate([x[..., half:], -x[..., :half]]"),
    "GQA grouping": ("kh = k[b, h // n_rep]", "kh = k[b, h % k.shape[1]]"),
    "eps outside the root": ("np.sqrt(mean_sq + eps)", "(np.sqrt(mean_sq) + eps)"),
    "mask hides the diagonal": ("np.where(kpos <= qpos, 0.0, -np.inf)", "np.where(kpos < qpos, 0.0, -np.inf)"),
    "score scale 1/d_h": ("scale = 1.0 / np.sqrt(dh)", "scale = 1.0 / dh"),
    "SiLU on up": ("return linear(silu(gate) * up, w_down)", "return linear(gate * silu(up), w_down)"),
    "inv_freq exponent": ("exps = np.arange(0, head_dim, 2, dtype=np.float64) / head_dim",
                          "exps = np.arange(0, head_dim, 2, dtype=np.float64) / (head_dim - 1)"),
    "decode position off by one": ("pos = np.full((1, 1, 1), float(L))", "pos = np.full((1, 1, 1), float(L + 1))"),
    "extend ignores the offset": ("pos = (L + np.arange(T, dtype=np.float64))[None, None, :]",
                                  "pos = (np.arange(T, dtype=np.float64))[None, None, :]"),
    "extend key order": ("K_all = np.concatenate([kc[:, :, :L], k], axis=2)",
                         "K_all = np.concatenate([k, kc[:, :, :L]], axis=2)"),
    "INT8 scale /128": ("s = (amax / np.float32(127.0)).astype(np.float32)",
                        "s = (amax / np.float32(128.0)).astype(np.float32)"),
    "INT8 truncation": ("q = np.rint(w32 / safe[:, None]).astype(np.float32)",
                        "q = np.trunc(w32 / safe[:, None]).astype(np.float32)"),
    "TP MLP without its norm": ('return swiglu_mlp(rmsnorm(X1, Ws["g_mlp"], eps), Ws["w_gate"], Ws["w_up"], Ws["w_down"])',
                                'return swiglu_mlp(X1, Ws["w_gate"], Ws["w_up"], Ws["w_down"])'),
    "stack passes X' on": ('        out = block_prefill(h, W, n_heads, n_kv_heads, head_dim, eps, rope_base)\n        h = out["y"]',
                           '        out = block_prefill(h, W, n_heads, n_kv_heads, head_dim, eps, rope_base)\n        h = out["x1"]'),
    "NTK exponent": ("return float(base) * s ** (head_dim / (head_dim - 2.0))",
                     "return float(base) * s ** (head_dim / (head_dim - 1.0))"),
    "NTK ratio": ("s = factor * L / L0 - (factor - 1.0)", "s = factor * L / L0"),
    "KV ledger without K+V": ("return layers * 2 * B * T * n_kv_heads * head_dim * dtype_bytes",
                              "return layers * B * T * n_kv_heads * head_dim * dtype_bytes"),
}


def main() -> int:
    src = open(os.path.join(ROOT, "oracle", "block.py")).read()
    survivors = []
    with tempfile.TemporaryDirectory() as tmp:
        for part in ("oracle", "tests", "synth"):
            shutil.copytree(os.path.join(ROOT, part), os.path.join(tmp, part),
                            ignore=shutil.ignore_patterns("__pycache__"))
        shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp)
        target = os.path.join(tmp, "oracle", "block.py")
        for name, (old, new) in MUTATIONS.items():
            if old not in src:
                print(f"{name:28s} STALE (the text to mutate is gone)")
                survivors.append(name)
                continue
            with open(target, "w") as f:
                f.write(src.replace(old, new, 1))
            r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle.py", "tests/test_tp_host.py",
                                "-q", "-x", "-m", "not gpu"], cwd=tmp, capture_output=True, text=True)
            caught = r.returncode != 0
            print(f"{name:28s} {'caught' if caught else 'SURVIVED'}", flush=True)
            if not caught:
                survivors.append(name)
    return 1 if survivors else 0


if __name__ == "__main__":
    sys.exit(main())
