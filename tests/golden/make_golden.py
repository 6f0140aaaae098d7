"""Writes the stored expected values under this folder.  It calls only the float64
oracle; nothing here comes from the library.  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import cag64  # noqa: E402


def growth_480p() -> dict:
    """Chunk-aware growth over a 7-chunk, 3-frames-per-chunk generation at the 480p shape
    (25 blocks of 64 tokens per frame, at most 6 frames retrieved).  The first chunk is
    dense; chunks 2-7 average 80% sparsity and chunk 7 sits at 90%: the two levels the
    article "南洋理工大学AI新突破 视频生成引擎模仿人脑高效学习" (m.youleyou.com) tests
    in section 一 (80% on chunks 2-7 after a dense first chunk; 90% as the harsher
    setting), put into the schedule s_i = s_base - alpha_i * beta of "Light Forcing:
    Accelerating Autoregressive Video Diffusion via Sparse Attention" (gist.science),
    section 2.1."""
    n, first, mean, final = 7, 2, 0.8, 0.9
    n_hist = [3 * i for i in range(n)]
    s, s_base, beta = cag64.cag_sparsity(n, first, mean, final)
    keep, budgets = cag64.cag_schedule(n, first, mean, final, n_hist, n_bpf=25, kf_max=6)
    return {
        "source": "oracle/cag64.py via tests/golden/make_golden.py",
        "citation": growth_480p.__doc__.strip().replace("\n    ", " "),
        "args": {"n_chunks": n, "first": first, "mean_sparsity": mean,
                 "final_sparsity": final, "n_hist": n_hist, "n_bpf": 25, "kf_max": 6},
        "s_base": s_base, "beta": beta, "sparsity": s, "keep": keep,
        "budgets": [list(b) for b in budgets],
    }


def main() -> None:
    path = os.path.join(HERE, "cag_growth_480p.json")
    with open(path, "w") as f:
        json.dump(growth_480p(), f, indent=1, ensure_ascii=False)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
