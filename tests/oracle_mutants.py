"""Plant mistakes in a copy of the oracle and check that its pins catch each.

    python tests/oracle_mutants.py [--workdir DIR] [NAME ...]

Each mutant is one plausible slip in ``oracle/hip_oracle.c`` (a wrong tie
rule, split point, representative block, reduction order, causal bound,
chunk tiling, reuse tail, dropped term, ...). The script copies the oracle,
the tests and the workload generator into a scratch directory, applies the
mutant there, runs ``tests/test_oracle_pins.py`` against the copy and reports
the first failing pin. A mutant that passes every pin is a gap in the pins;
the exit status is the number of such survivors, plus the number of mutants
whose target text no longer occurs exactly once in the oracle (reported as
STALE and counted as not caught). Nothing in the repository itself is
modified.
"""
import argparse
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text in hip_oracle.c, replacement)
MUTANTS = [
    ("tie_rule", "return (a->s > b->s) - (a->s < b->s);",
     "return (a->s < b->s) - (a->s > b->s);"),
    ("representative", "int64_t rep = cands[c].s + (cands[c].e - cands[c].s) / 2;",
     "int64_t rep = cands[c].s + (cands[c].e - cands[c].s - 1) / 2;"),
    ("split_point", "int64_t m = s + L / 2;", "int64_t m = s + (L + 1) / 2;"),
    ("tree_order", "float a0 = part[0] + part[4], a1 = part[1] + part[5];",
     "float a0 = part[0] + part[1], a1 = part[4] + part[5];"),
    ("causal_bound", "if (j > p) continue;", "if (j > p + 1) continue;"),
    ("chunk_tiling", "chunks[i].s = i * N / n0;\n      chunks[i].e = (i + 1) * N / n0;",
     "chunks[i].s = (i * N + n0 - 1) / n0;\n      chunks[i].e = ((i + 1) * N + n0 - 1) / n0;"),
    ("reuse_tail",
     "for (int64_t j = sh->mask_len; j < sh->seq_len && j <= p; ++j) keys[n++] = j;",
     "for (int64_t j = sh->mask_len; j + 1 < sh->seq_len && j <= p; ++j) keys[n++] = j;"),
    ("dropped_dot_term", "for (int e = 0; e < 8; ++e) acc = fmaf",
     "for (int e = 0; e < 7; ++e) acc = fmaf"),
    ("sink_floor", "c < min64(cdiv64(sh->sink, bk), N)", "c < min64(sh->sink / bk, N)"),
    ("window_from_last", "int64_t lo = max64(0, q_first - sh->window + 1);",
     "int64_t lo = max64(0, q_last - sh->window + 1);"),
    ("score_last_not_max", "if (sc > best) best = sc;", "best = sc;"),
    ("attn_scale", "const double scale = 1.0 / sqrt((double)d);",
     "const double scale = 1.0 / sqrt((double)d + 1);"),
    ("attn_drop_first_weight", "    l += w;\n", "    l += (t ? w : 0.0);\n"),
    ("gqa_head", "u->h0 = sh->per_head ? hm : hm * G;", "u->h0 = sh->per_head ? hm : hm;"),
    ("stop_early", "if (longest <= 1 && nk <= n0) break;", "if (longest <= 2 && nk <= n0) break;"),
    ("stage_keep_count", "const int64_t m = g->stage_k / g->chunk_size;",
     "const int64_t m = g->stage_k / g->chunk_size + 1;"),
    ("stage_rows_from_first", "for (int64_t i = u->i1 - 1; i >= u->i0; i -= stride) {",
     "for (int64_t i = u->i0; i < u->i1; i += stride) {"),
    ("stage_chunk_in_keys", "const int64_t cs = g->chunk_size / bk;",
     "const int64_t cs = g->chunk_size;"),
    ("stage_stride_dropped", "                                       g->stride_q);",
     "                                       1);"),
    ("stage_rep_start", "cands[c].score = block_score(q, k, sh, &u, cands[c].s + (cands[c].e - cands[c].s) / 2,",
     "cands[c].score = block_score(q, k, sh, &u, cands[c].s + (cands[c].e - cands[c].s - 1) / 2,"),
    ("single_blocks_over_budget", "if (longest <= 1 && nk <= n0) break;", "if (longest <= 1) break;"),
    ("per_head_kv_map", "u->g = sh->per_head ? hm / G : hm;",
     "u->g = sh->per_head ? hm % sh->n_kvheads : hm;"),
    ("per_head_idx_row", "const int64_t mrow = sh->per_head ? b * sh->n_qheads + h : b * sh->n_kvheads + g;",
     "const int64_t mrow = sh->per_head ? b * sh->n_qheads + g : b * sh->n_kvheads + g;"),
    ("e5m2_bias", "v = ldexp(1.0 + m / 4.0, e - 15);", "v = ldexp(1.0 + m / 4.0, e - 16);"),
    ("e5m2_subnormal", "v = ldexp(m / 4.0, -14);", "v = ldexp(1.0 + m / 4.0, -15);"),
    ("e5m2_mantissa", "const int sign = c >> 7, e = (c >> 2) & 31, m = c & 3;",
     "const int sign = c >> 7, e = (c >> 2) & 31, m = (c >> 1) & 3;"),
]


def stale_targets(text=None):
    """Names of the mutants whose target text does not occur exactly once."""
    if text is None:
        with open(os.path.join(ROOT, "oracle", "hip_oracle.c")) as f:
            text = f.read()
    return [name for name, old, _ in MUTANTS if text.count(old) != 1]


def run_one(name, old, new, workdir):
    d = os.path.join(workdir, name)
    if os.path.exists(d):
        shutil.rmtree(d)
    os.makedirs(d)
    for sub in ("oracle", "tests", "hierarchically_pruned_sparse_b200"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub),
                        ignore=shutil.ignore_patterns("*.so", "*.so.*", "__pycache__", "_build"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), d)
    src = os.path.join(d, "oracle", "hip_oracle.c")
    text = open(src).read()
    if text.count(old) != 1:
        shutil.rmtree(d)
        return False, f"STALE: its target text occurs {text.count(old)} times in the oracle"
    open(src, "w").write(text.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=d, capture_output=True, text=True)
    shutil.rmtree(d)
    failed = [ln for ln in r.stdout.splitlines() if ln.startswith("FAILED")]
    return r.returncode != 0, (failed[0] if failed else r.stdout.strip().splitlines()[-1])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workdir", default=None)
    ap.add_argument("names", nargs="*")
    args = ap.parse_args()
    workdir = args.workdir or tempfile.mkdtemp(prefix="oracle_mutants_")
    os.makedirs(workdir, exist_ok=True)
    survivors = 0
    for name, old, new in MUTANTS:
        if args.names and name not in args.names:
            continue
        caught, first = run_one(name, old, new, workdir)
        survivors += not caught
        print(f"{name:24s} {'caught' if caught else 'SURVIVED'}  {first}", flush=True)
    return survivors


if __name__ == "__main__":
    sys.exit(main())
