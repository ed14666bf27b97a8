"""Plant plausible mistakes in copies of the CPU oracle and check that the pins
catch every one. The committed oracle source is never modified: each mutant is
a textual copy compiled into a temporary library."""
import os

import pytest

import oracle
import pins

# (what the mistake is, text in lsa_oracle.c, replacement)
MUTANTS = [
    ("fine score drops the ReLU", "        if (dot > 0)\n            total += (int64_t)w[h] * dot;\n    }\n    return total;\n}\n\n/* Per-block",
     "        total += (int64_t)w[h] * dot;\n    }\n    return total;\n}\n\n/* Per-block"),
    ("fine score ReLU with the wrong sign", "        if (dot > 0)\n            total += (int64_t)w[h] * dot;\n    }\n    return total;\n}\n\n/* Per-block",
     "        if (dot < 0)\n            total += (int64_t)w[h] * dot;\n    }\n    return total;\n}\n\n/* Per-block"),
    ("fine score reads the wrong head weight", "            total += (int64_t)w[h] * dot;\n    }\n    return total;\n}\n\n/* Per-block",
     "            total += (int64_t)w[0] * dot;\n    }\n    return total;\n}\n\n/* Per-block"),
    ("fine score transposes q", "            dot += (int64_t)q[h * d_I + d] * (int64_t)k[d];",
     "            dot += (int64_t)q[d * H_I + h] * (int64_t)k[d];"),
    ("block sums shifted by one token", "        int64_t b = t / B;", "        int64_t b = (t + B - 1) / B < nblk ? (t + B - 1) / B : nblk - 1;"),
    ("coarse score drops the ReLU", "            dot += (int64_t)q[h * d_I + d] * S_b[d];\n        if (dot > 0)",
     "            dot += (int64_t)q[h * d_I + d] * S_b[d];\n        if (1)"),
    ("ties go to the higher position", "    return x->pos < y->pos ? -1 : (x->pos > y->pos ? 1 : 0);",
     "    return x->pos > y->pos ? -1 : (x->pos < y->pos ? 1 : 0);"),
    ("ascending score order", "        return x->score > y->score ? -1 : 1;", "        return x->score < y->score ? -1 : 1;"),
    ("window one token short", "    int64_t ws = L - window > s ? L - window : s;", "    int64_t ws = L - window + 1 > s ? L - window + 1 : s;"),
    ("sink not clipped to the context", "    int64_t s = sink < L ? sink : L;", "    int64_t s = sink;"),
    ("top-k one short", "    int64_t n_sel = n_cand < topk ? n_cand : topk;", "    int64_t n_sel = n_cand < topk ? n_cand : (topk > 0 ? topk - 1 : 0);"),
    ("HI candidate blocks exclude the sink block", "            if (lo < ws && hi > s) {", "            if (lo >= s && lo < ws && hi > s) {"),
    ("HI keeps one block too few", "        int64_t keep = n_cb < hi_topblocks ? n_cb : hi_topblocks;",
     "        int64_t keep = n_cb < hi_topblocks ? n_cb : (hi_topblocks > 0 ? hi_topblocks - 1 : 0);"),
    ("softmax scale 1/d", "    double scale = 1.0 / sqrt((double)d);", "    double scale = 1.0 / (double)d;"),
    ("GQA interleaved instead of contiguous", "        int kvh = (int)(((int64_t)h * H_kv) / H_q);", "        int kvh = h % H_kv;"),
    ("softmax not normalised", "            out[h * d + e] /= denom;", "            out[h * d + e] /= 1.0;"),
    ("attention uses K for V", "            const uint16_t *vrow = vseq + ((int64_t)set[j] * H_kv + kvh) * d;",
     "            const uint16_t *vrow = kseq + ((int64_t)set[j] * H_kv + kvh) * d;"),
    ("batch driver ignores the sequence offset", "        const int8_t *kseq = j->k_idx + j->kv_offset[j->q_seq[r]] * j->d_I;",
     "        const int8_t *kseq = j->k_idx;"),
    ("batch driver gives every row the first row's weights", "        int n = oracle_index_query(j->q_idx + r * j->H_I * j->d_I, j->w + r * j->H_I,",
     "        int n = oracle_index_query(j->q_idx + r * j->H_I * j->d_I, j->w,"),
    ("batch driver sees one token fewer", "                                   kseq, j->q_len[r], j->H_I, j->d_I, j->sink,",
     "                                   kseq, j->q_len[r] - 1, j->H_I, j->d_I, j->sink,"),
    ("E4M3 exponent bias 8", "        v = ldexp(1.0 + (double)m / 8.0, E - 7);", "        v = ldexp(1.0 + (double)m / 8.0, E - 8);"),
    ("E4M3 subnormals read as normals", "        v = ldexp((double)m / 8.0, -6);", "        v = ldexp(1.0 + (double)m / 8.0, -6);"),
    ("E4M3 sign dropped", "    return sign ? -v : v;", "    return v;"),
    ("FP8 attention ignores the K scale",
     "                dot += bf16_to_double(q[h * d + e]) * (k_scale * oracle_e4m3_value(krow[e]));",
     "                dot += bf16_to_double(q[h * d + e]) * oracle_e4m3_value(krow[e]);"),
    ("FP8 attention scales V by the K scale",
     "                out[h * d + e] += p * (v_scale * oracle_e4m3_value(vrow[e]));",
     "                out[h * d + e] += p * (k_scale * oracle_e4m3_value(vrow[e]));"),
    ("FP8 attention softmax scale 1/d", "    const double inv_sqrt_d = 1.0 / sqrt((double)d);",
     "    const double inv_sqrt_d = 1.0 / (double)d;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {name}"
    lib = oracle.build(output=str(tmp_path / "mutant.so"), source_text=src.replace(old, new))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
        except (ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught: {name}"
