"""Plant plausible mistakes in a COPY of the oracle's C source and check that the
pins catch every one (CPU only).  The committed oracle is never modified; each
planted copy is compiled into a temporary directory and loaded on its own."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "tf_oracle.c")

# (name, original text, planted text).  Each planted copy reads only inside its
# buffers (no out-of-range positions), so a failing pin is an assertion, not a crash.
PLANTS = [
    ("gqa mapping by modulo", "const int32_t kh = h / J->G;", "const int32_t kh = h % J->Hkv;"),
    ("window one position early", "return j <= base + r;", "return j <= base + r - 1;"),
    ("window ignores row index", "return j <= base + r;", "return j <= base;"),
    ("softmax sign flipped", "w[j] = exp(x[j] - mx);", "w[j] = exp(mx - x[j]);"),
    ("scale dropped", "x[j] = J->scale * acc;", "x[j] = acc;"),
    ("no normalisation", "o[i] /= l;", "o[i] /= 1.0;"),
    ("values read from keys", "const uint16_t *vs = J->v + J->kv_off[s];",
     "const uint16_t *vs = J->k + J->kv_off[s];"),
    ("query rows transposed", "(((int64_t)s * J->W + r) * Hq + h) * d;",
     "(((int64_t)s * Hq + h) * J->W + r) * d;"),
    ("key cache read head-major", "const uint16_t *krow = ks + (pos[j] * J->Hkv + kh) * d;",
     "const uint16_t *krow = ks + ((int64_t)kh * J->lens[s] + pos[j]) * d;"),
    ("last key dropped from the sum", "for (j = 0; j < n; ++j) {\n        w[j]",
     "for (j = 0; j < n - 1; ++j) {\n        w[j]"),
    ("tree bit taken by row, not key", "return (J->tree[(int64_t)s * J->W + r] >> (j - base)) & 1;",
     "return (J->tree[(int64_t)s * J->W + r] >> r) & 1;"),
    ("tree mask of the mirrored row", "return (J->tree[(int64_t)s * J->W + r] >> (j - base)) & 1;",
     "return (J->tree[(int64_t)s * J->W + (J->W - 1 - r)] >> (j - base)) & 1;"),
    ("tree mask shifted by one key", "return (J->tree[(int64_t)s * J->W + r] >> (j - base)) & 1;",
     "return (J->tree[(int64_t)s * J->W + r] >> (j - base + 1)) & 1;"),
    ("copy destination slot off by one",
     "const int64_t to = (((int64_t)dp * Hkv + kh) * dst_P + j % dst_P) * d;",
     "const int64_t to = (((int64_t)dp * Hkv + kh) * dst_P + (j + 1) % dst_P) * d;"),
    ("copy drops the last position", "for (j = 0; j < lens[s]; ++j) {\n            const int32_t sp",
     "for (j = 0; j + 1 < lens[s]; ++j) {\n            const int32_t sp"),
    ("copy reads the mirrored KV head",
     "const int64_t from = (((int64_t)sp * Hkv + kh) * src_P + j % src_P) * d;",
     "const int64_t from = (((int64_t)sp * Hkv + (Hkv - 1 - kh)) * src_P + j % src_P) * d;"),
    ("row write slot off by one", "const int64_t slot = pos % P;",
     "const int64_t slot = (pos + 1) % P;"),
    ("row write pool index transposed", "(((int64_t)page * Hkv + kh) * P + slot) * d;",
     "(((int64_t)kh * n_pages + page) * P + slot) * d;"),
]


@pytest.mark.parametrize("name,orig,planted", PLANTS, ids=[p[0] for p in PLANTS])
def test_pins_catch_planted_mistake(tmp_path, name, orig, planted):
    text = open(SRC).read()
    assert text.count(orig) == 1, f"plant site for {name!r} not found exactly once"
    src = tmp_path / "planted.c"
    src.write_text(text.replace(orig, planted))
    lib = oracle.open_library(oracle.compile_source(str(src), str(tmp_path / "libplanted.so")))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib=lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name!r}"
