"""The pins must catch plausible mistakes in the oracle.

Each case copies oracle.c to a temporary directory, plants one mistake (a wrong sign,
a dropped term, a wrong index, a swapped operand), compiles it, and runs the pin suite
against that build on the CPU. The suite must fail. Nothing here touches a GPU."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTATIONS = {
    "rope_sign": ("x[i] = x0 * c - x1 * s;", "x[i] = x0 * c + x1 * s;"),
    "rope_frequency": ("pow(base, -2.0 * (double)i / (double)d)", "pow(base, -1.0 * (double)i / (double)d)"),
    "rope_adjacent_pairing": ("double x0 = x[i], x1 = x[i + half];\n            x[i] = x0 * c - x1 * s;\n"
                              "            x[i + half] = x0 * s + x1 * c;",
                              "double x0 = x[2 * i], x1 = x[2 * i + 1];\n            x[2 * i] = x0 * c - x1 * s;\n"
                              "            x[2 * i + 1] = x0 * s + x1 * c;"),
    "causal_drops_current_token": ("d, first, pos + 1,", "d, first, pos,"),
    "gqa_interleaved_mapping": ("        int g = hh / group;\n        orc_attend_window(q + (int64_t)hh * d, K0",
                                "        int g = hh % nkv;\n        orc_attend_window(q + (int64_t)hh * d, K0"),
    "rmsnorm_no_eps": ("acc / (double)n + eps", "acc / (double)n"),
    "attention_no_scale": ("s[j] = acc * scale;", "s[j] = acc;"),
    "silu_is_sigmoid": ("return z * (1.0 / (1.0 + exp(-z)));", "return (1.0 / (1.0 + exp(-z)));"),
    "gate_up_swapped": ("g[i] = orc_bf16(silu(g[i]) * u[i]);", "g[i] = orc_bf16(silu(u[i]) * g[i]);"),
    "no_r4_rounding": ("g[i] = orc_bf16(silu(g[i]) * u[i]);", "g[i] = silu(g[i]) * u[i];"),
    "no_r1_rounding": ("    for (int i = 0; i < h; ++i) xn[i] = orc_bf16(xn[i]);\n    /* 2.",
                       "    /* 2."),
    "renorm_ignored": ("w[r] = renorm ? p[order[r]] / sum : p[order[r]];", "w[r] = p[order[r]];"),
    "shared_gate_no_sigmoid": ("sc = sigmoid(gdot);", "sc = gdot;"),
    "tie_break_higher_index": ("(best < 0 || p[e] > p[best])", "(best < 0 || p[e] >= p[best])"),
    "residual_dropped": ("post_attn_norm, h, c->eps, t);\n    for (int i = 0; i < h; ++i) x[i] += t[i];",
                         "post_attn_norm, h, c->eps, t);\n    for (int i = 0; i < h; ++i) x[i] = t[i];"),
    "qkv_bias_dropped": ("qkv[r] += (double)L->bqkv[r];", "qkv[r] += 0.0;"),
    "cache_row_off_by_one": ("uint16_t* krow = kslot(m, m->kc, seq, li, pos);",
                             "uint16_t* krow = kslot(m, m->kc, seq, li, pos + 1 < m->c.max_ctx ? pos + 1 : pos);"),
    "qk_norm_after_rope": ("""    if (c->qk_norm) {
        orc_head_rmsnorm(q, nq, d, L->q_norm, c->eps);
        orc_head_rmsnorm(k, nkv, d, L->k_norm, c->eps);
    }
    /* 4. RoPE on q and k at pos */
    orc_rope(q, nq, d, pos, c->rope_base);
    orc_rope(k, nkv, d, pos, c->rope_base);""", """    orc_rope(q, nq, d, pos, c->rope_base);
    orc_rope(k, nkv, d, pos, c->rope_base);
    if (c->qk_norm) {
        orc_head_rmsnorm(q, nq, d, L->q_norm, c->eps);
        orc_head_rmsnorm(k, nkv, d, L->k_norm, c->eps);
    }"""),
    "qk_norm_gains_swapped": ("""        orc_head_rmsnorm(q, nq, d, L->q_norm, c->eps);
        orc_head_rmsnorm(k, nkv, d, L->k_norm, c->eps);""", """        orc_head_rmsnorm(q, nq, d, L->k_norm, c->eps);
        orc_head_rmsnorm(k, nkv, d, L->q_norm, c->eps);"""),
    "qk_norm_whole_vector": ("""    for (int hh = 0; hh < heads; ++hh) orc_rmsnorm(v + (int64_t)hh * d, g, d, eps, v + (int64_t)hh * d);""",
                             """    double acc = 0.0;
    for (int64_t i = 0; i < (int64_t)heads * d; ++i) acc += v[i] * v[i];
    double inv = 1.0 / sqrt(acc / ((double)heads * d) + eps);
    for (int64_t i = 0; i < (int64_t)heads * d; ++i) v[i] = v[i] * inv * (double)g[i % d];"""),
    "qk_norm_bias_after_norm": ("""    if (c->qkv_bias && L->bqkv)
        for (int64_t r = 0; r < rows; ++r) qkv[r] += (double)L->bqkv[r];
    double* q = qkv;
    double* k = qkv + qd;
    double* v = qkv + qd + kvd;
    /* 3. optional per-head QK-norm (applyHeadNorm): q heads with q_norm, k heads with k_norm */
    if (c->qk_norm) {
        orc_head_rmsnorm(q, nq, d, L->q_norm, c->eps);
        orc_head_rmsnorm(k, nkv, d, L->k_norm, c->eps);
    }""", """    double* q = qkv;
    double* k = qkv + qd;
    double* v = qkv + qd + kvd;
    if (c->qk_norm) {
        orc_head_rmsnorm(q, nq, d, L->q_norm, c->eps);
        orc_head_rmsnorm(k, nkv, d, L->k_norm, c->eps);
    }
    if (c->qkv_bias && L->bqkv)
        for (int64_t r = 0; r < rows; ++r) qkv[r] += (double)L->bqkv[r];"""),
    "window_one_key_too_many": ("pos + 1 > window ? pos + 1 - window : 0;", "pos + 1 > window ? pos - window : 0;"),
    "window_schedule_inverted": ("(layer + 1) % pattern != 0 ? c->sliding_window : 0",
                                 "(layer + 1) % pattern == 0 ? c->sliding_window : 0"),
    "softcap_before_scale": ("""        s[j] = acc * scale;
        if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);""",
                             """        s[j] = (softcap > 0.0 ? softcap * tanh(acc / softcap) : acc) * scale;"""),
    "softcap_ignored": ("        if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);\n", ""),
    "sandwich_post_attn_dropped": ("    if (c->sandwich) orc_rmsnorm(t, L->post_attn_norm, h, c->eps, t);\n", ""),
    "sandwich_ffn_uses_attn_gain": ("orc_rmsnorm(t, L->post_ffn_norm,", "orc_rmsnorm(t, L->post_attn_norm,"),
    "final_softcap_dropped": ("logits[v] = c->final_softcap * tanh(logits[v] / c->final_softcap);",
                              "logits[v] = logits[v];"),
    "q8_scale_ignored": ("acc += (sc * (double)q[k]) * x[k];", "acc += ((double)q[k]) * x[k];"),
    "q8_first_row_scale": ("const double sc = (double)S[n];", "const double sc = (double)S[0];"),
    "tied_head_ignored": ("const uint16_t* head = c->tied ? m->w.embed : m->w.lm_head;",
                          "const uint16_t* head = m->w.embed;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    c_file = tmp_path / "oracle.c"
    c_file.write_text(mutated)
    (tmp_path / "oracle.h").write_text(open(os.path.join(ROOT, "oracle", "oracle.h")).read())
    so = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-o", str(so),
                           str(c_file), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(so), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"
