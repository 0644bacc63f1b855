"""The oracle's pins are sensitive: each plausible mistake planted in a copy
of the oracle source (on the CPU, in a temporary directory) makes at least one
pin of ``test_oracle_pieces.py`` / ``test_oracle_invariants.py`` fail.

Each mutant is a single textual edit of ``oracle/rlt_oracle.c``; the edit must
apply exactly once, so the list stays in step with the source.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "rlt_oracle.c")

MUTANTS = {
    "gate bias dropped": ("orc_sigmoid(gpre[i] + w->gate_b[i])", "orc_sigmoid(gpre[i])"),
    "gate concat order swapped": ("cat[i] = e_t[i];\n    cat[d + i] = s_prev[i];",
                                  "cat[i] = s_prev[i];\n    cat[d + i] = e_t[i];"),
    "feedback scale ignored": ("(real)c->alpha * g * s_prev[i]", "g * s_prev[i]"),
    "rotary sign flipped": ("v[i] = a * c - b * s;", "v[i] = a * c + b * s;"),
    "rotary frequency halved": ("pow(theta, -2.0 * i / dh)", "pow(theta, -1.0 * i / dh)"),
    "norm gain dropped": ("y[i] = x[i] * r * gamma[i];", "y[i] = x[i] * r;"),
    "norm epsilon dropped": ("(double)(ss / n) + eps", "(double)(ss / n)"),
    "attention scale 1/dh": ("1.0 / sqrt((double)dh)", "1.0 / (double)dh"),
    "gelu tanh form": ("return (real)(0.5 * x * (1.0 + erf(x / sqrt(2.0))));",
                       "return (real)(0.5 * x * (1.0 + tanh(0.7978845608 * (x + 0.044715 * x * x * x))));"),
    "s_t is the raw residual": ("orc_rmsnorm(h, w->dec_lnf, d, c->rms_eps, s);\n}",
                                "memcpy(s, h, sizeof(real) * d);\n}"),
    "memory prefix exclusive": ("s->vp, (int)t + 1, dh, s->sc", "s->vp, (int)t + (t == 0), dh, s->sc"),
    "memory group ignored": ("int g = (c->mem_groups == 1) ? 0 : l;", "int g = 0;"),
    "ffn reads the cross-attention norm": ("orc_rmsnorm(h, w->dec_ln3[l]", "orc_rmsnorm(h, w->dec_ln2[l]"),
    "window drops the current token": ("sc->kp[n] = sc->kcur + hd * dh;",
                                        "sc->kp[n] = n > 0 ? sc->kp[n - 1] : sc->kcur + hd * dh;"),
    "window one entry short": ("long nh = t < Wm1 ? t : Wm1;", "long nh = t < Wm1 - 1 ? t : (Wm1 > 0 ? Wm1 - 1 : 0);"),
    "encoder sees the future": (
        "for (int j = 0; j <= t; j++) {\n          kp[j] = qkv + (size_t)j * 3 * d + d + hd * dh;\n"
        "          vp[j] = qkv + (size_t)j * 3 * d + 2 * d + hd * dh;\n        }\n"
        "        orc_attend(qkv + (size_t)t * 3 * d + hd * dh, kp, vp, t + 1, dh, sc,",
        "for (int j = 0; j < T; j++) {\n          kp[j] = qkv + (size_t)j * 3 * d + d + hd * dh;\n"
        "          vp[j] = qkv + (size_t)j * 3 * d + 2 * d + hd * dh;\n        }\n"
        "        orc_attend(qkv + (size_t)t * 3 * d + hd * dh, kp, vp, T, dh, sc,"),
    "encoder key not rotated": ("orc_rope(qkv + (size_t)t * 3 * d + d + hd * dh, dh, t, c->rope_theta);",
                                "(void)0;"),
    "value projection rows shifted": ("memcpy(s->vcur, s->q + 2 * d, sizeof(real) * d);",
                                      "memcpy(s->vcur, s->q + d, sizeof(real) * d);"),
    "swiglu factors swapped": ("tmp_a[i] = orc_silu(tmp_a[i]) * tmp_b[i];",
                               "tmp_a[i] = tmp_a[i] * orc_silu(tmp_b[i]);"),
    "start state zero": ("memcpy(s, w->sstar, sizeof(real) * c->d);", "memset(s, 0, sizeof(real) * c->d);"),
    "encoder ffn reads the attention norm": (
        "orc_rmsnorm(h + (size_t)t * d, w->enc_ln2[l], d, c->rms_eps, u);",
        "orc_rmsnorm(h + (size_t)t * d, w->enc_ln1[l], d, c->rms_eps, u);"),
    "encoder ffn residual dropped": (
        "ffn(c, w->enc_w1[l], w->enc_wb[l], w->enc_w2[l], u, o, ta, tb);\n"
        "      for (int i = 0; i < d; i++) h[(size_t)t * d + i] += o[i];",
        "ffn(c, w->enc_w1[l], w->enc_wb[l], w->enc_w2[l], u, o, ta, tb);\n"
        "      for (int i = 0; i < d; i++) h[(size_t)t * d + i] = o[i];"),
    "encoder blocks reuse block 0's ffn": ("ffn(c, w->enc_w1[l], w->enc_wb[l], w->enc_w2[l],",
                                           "ffn(c, w->enc_w1[0], w->enc_wb[0], w->enc_w2[0],"),
    "encoder blocks reuse block 0's q/k/v": (
        "orc_linear(w->enc_wqkv[l], u, 3 * d, d, qkv + (size_t)t * 3 * d);",
        "orc_linear(w->enc_wqkv[0], u, 3 * d, d, qkv + (size_t)t * 3 * d);"),
    "decoder q/k/v of layer 0": ("orc_linear(w->dec_wqkv[l], s->u, 3 * d, d, s->q);",
                                 "orc_linear(w->dec_wqkv[0], s->u, 3 * d, d, s->q);"),
    "decoder output projection of layer 0": ("orc_linear(w->dec_wo[l], sc->a, d, d, sc->o);",
                                             "orc_linear(w->dec_wo[0], sc->a, d, d, sc->o);"),
    "decoder cross-attention query of layer 0": ("orc_linear(w->dec_wqx[l], s->u, d, d, s->q);",
                                                 "orc_linear(w->dec_wqx[0], s->u, d, d, s->q);"),
    "decoder cross-attention output of layer 0": ("orc_linear(w->dec_wox[l], s->a, d, d, s->o);",
                                                  "orc_linear(w->dec_wox[0], s->a, d, d, s->o);"),
    "decoder ffn of layer 0": ("ffn(c, w->dec_w1[l], w->dec_wb[l], w->dec_w2[l],",
                               "ffn(c, w->dec_w1[0], w->dec_wb[0], w->dec_w2[0],"),
    "sampler keeps the last maximum": ("if (logits[v] > logits[arg]) arg = v;",
                                       "if (logits[v] >= logits[arg]) arg = v;"),
    "sampler total weight at the inverse temperature": (
        "for (int v = 0; v < V; v++) Z += exp(((double)logits[v] - (double)logits[arg]) / tau);",
        "for (int v = 0; v < V; v++) Z += exp(((double)logits[v] - (double)logits[arg]) * tau);"),
    "lm head reads s at an offset": ("orc_linear(w->embed, s, c->vocab, c->d, logits);",
                                     "orc_linear(w->embed + 1, s, c->vocab - 1, c->d, logits);"),
    "decoder cross-attention norms in reverse layer order": (
        "orc_rmsnorm(h, w->dec_ln2[l], d, c->rms_eps, s->u);",
        "orc_rmsnorm(h, w->dec_ln2[c->n_dec - 1 - l], d, c->rms_eps, s->u);"),
}

PIN_FILES = ["tests/test_oracle_pieces.py", "tests/test_oracle_invariants.py"]


def _build_and_run(name, edit, tmp):
    old, new = edit
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutant '{name}' no longer applies"
    stem = "".join(ch if ch.isalnum() else "_" for ch in name)
    path = os.path.join(tmp, stem + ".c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = path[:-2] + ".so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                           "-DORC_REAL=double", path, "-o", so, "-lm"])
    env = dict(os.environ, RLT_ORACLE_LIB_F64=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PIN_FILES], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
            futs = {n: ex.submit(_build_and_run, n, e, tmp) for n, e in MUTANTS.items()}
            codes = {n: f.result() for n, f in futs.items()}
    survived = [n for n, c in codes.items() if c == 0]
    assert not survived, f"planted mistakes no pin caught: {survived}"
    assert all(c == 1 for c in codes.values()), codes
