"""Pins the oracle to the printed output of the demo on page "How does a tree of
summaries search a context? How ZHA works", section "Run a small tree yourself".

The demo's workload is restated in tests/demo_tree.c (JavaScript number semantics);
all tree arithmetic (summaries, walk, work count, kept attention) is the oracle's.
The printed integers (mean comparisons per query and mean % of attention kept, for
1K..64K keys) must come out exactly. A second test plants plausible mistakes in a
copy of the oracle and checks that each one changes the printed numbers, so that
the pin really constrains those parts of the oracle.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
GOLDEN = os.path.join(HERE, "golden", "demo_tree_output.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


def _run(tmp, oracle_src, store=1):
    os.makedirs(os.path.join(tmp, "oracle"), exist_ok=True)
    os.makedirs(os.path.join(tmp, "tests"), exist_ok=True)
    shutil.copy(os.path.join(ROOT, "oracle", "zha_oracle.h"), os.path.join(tmp, "oracle"))
    with open(os.path.join(tmp, "oracle", "zha_oracle.c"), "w") as f:
        f.write(oracle_src)
    shutil.copy(os.path.join(HERE, "demo_tree.c"), os.path.join(tmp, "tests"))
    exe = os.path.join(tmp, "demo_tree")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-o", exe,
                    os.path.join(tmp, "tests", "demo_tree.c"), os.path.join(tmp, "oracle", "zha_oracle.c"),
                    "-lm"], check=True)
    out = subprocess.run([exe, str(store)], check=True, capture_output=True, text=True).stdout
    return [tuple(int(x) for x in line.split()) for line in out.strip().splitlines()]


def _src():
    with open(os.path.join(ROOT, "oracle", "zha_oracle.c")) as f:
        return f.read()


@pytest.mark.parametrize("store", [1, 3, 0], ids=["demo_f32_keys", "f32_keys_and_bias", "f64"])
def test_demo_output_reproduced(tmp_path, store):
    # store 1 = keys fp32, biases double (as the demo keeps them); 3 = both fp32
    # (as the CUDA library stores nodes); 0 = nothing rounded.
    assert _run(str(tmp_path), _src(), store) == _golden()


MUTATIONS = {
    # a wrong sign on the child bias inside a summary
    "child_bias_sign": ("s[i] = beta * dot(k, q, d) + b;", "s[i] = beta * dot(k, q, d) - b;"),
    # the bias correction of a summary dropped (bias = logsumexp only)
    "bias_correction_dropped": ("log_sum_exp(s, n_children) - beta * dot(key, q, d)",
                                "log_sum_exp(s, n_children)"),
    # plain averaging of the children instead of the softmax weights
    "mean_instead_of_softmax": ("acc[t] += w[i] * k[t];", "acc[t] += k[t] / n_children;"),
    # the node's bias left out of the walk's score
    "walk_score_without_bias": ("query, d) + bias[F[i] * R + r];", "query, d);"),
    # the reference index dropped when reading a node key in the walk
    "walk_key_index": ("keys + (F[i] * R + r) * d", "keys + (F[i] * R) * d"),
    # the comparisons counted once per node instead of once per reference
    "work_per_node": ("*work = (long long)R * total_frontier", "*work = total_frontier"),
    # the top-p prefix stopping one node early
    "top_p_one_short": ("if (total >= p) {", "if (total + rk[c - 1].mass >= p) {"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_breaks_the_pin(tmp_path, name):
    old, new = MUTATIONS[name]
    src = _src()
    assert old in src, f"mutation site for {name} not found"
    assert _run(str(tmp_path), src.replace(old, new)) != _golden()
