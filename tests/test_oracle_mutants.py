"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one (CPU only).  The real oracle file is never modified: each
mutant is an edited copy compiled into a temporary library."""
import pytest

import oracle as O
from tests import oracle_pins as P

MUTANTS = [
    ("scale dropped", "s[r] = dot * scale;", "s[r] = dot;"),
    ("tie break reversed", "return (a->i < b->i) ? -1 : (a->i > b->i) ? 1 : 0;",
     "return (a->i > b->i) ? -1 : (a->i < b->i) ? 1 : 0;"),
    ("selection left in value order", "qsort(S, (size_t)keff, sizeof(int32_t), by_int_asc);", ""),
    ("wrong GQA group", "const int g = h / G;\n      const int64_t kv_base",
     "const int g = h % Hkv;\n      const int64_t kv_base"),
    ("sparse head reads every row", "attend_rows(sh, q, K, V, kv_base, S, count, o, NULL);",
     "attend_rows(sh, q, K, V, kv_base, NULL, n, o, NULL);"),
    ("never refreshed after layer 0", "if (!fresh[s]) {", "if (!fresh[s] || l > 0) {"),
    ("group mean over the wrong heads", "(((int64_t)l * B + b) * Hq + (g * G + t)) * d;",
     "(((int64_t)l * B + b) * Hq + (t)) * d;"),
    ("logits against V", "for (int j = 0; j < d; ++j) dot += q[j] * widen(K, sh->dtype, off + j);",
     "for (int j = 0; j < d; ++j) dot += q[j] * widen(V, sh->dtype, off + j);"),
    ("layer-0 rule dropped", "is_ret[h] = all_retrieval || role_row[h] != 0;",
     "is_ret[h] = role_row[h] != 0;"),
    ("padding not -1", "for (int64_t j = keff; j < k; ++j) S[j] = -1;",
     "for (int64_t j = keff; j < k; ++j) S[j] = 0;"),
    ("last inherited row dropped", "while (count < k && S[count] >= 0) ++count;",
     "while (count < k - 1 && S[count] >= 0) ++count;"),
    ("bf16 widened with the wrong shift", "uint32_t bits = ((uint32_t)h) << 16;",
     "uint32_t bits = ((uint32_t)h) << 15;"),
    ("softmax not normalised", "for (int j = 0; j < d; ++j) o[j] /= z;", ""),
    ("token stride ignored", "int64_t off = kv_base + i * sh->s_token;\n    double dot",
     "int64_t off = kv_base + i * sh->d;\n    double dot"),
    ("value row from the wrong token",
     "for (int j = 0; j < d; ++j) o[j] += p * widen(V, sh->dtype, off + j);",
     "for (int j = 0; j < d; ++j) o[j] += p * widen(V, sh->dtype, kv_base + r * sh->s_token + j);"),
    ("ratio rounded down", "int64_t m = (sel->ratio_num * n + sel->ratio_den - 1) / sel->ratio_den;",
     "int64_t m = (sel->ratio_num * n) / sel->ratio_den;"),
    ("top-p takes one row too many", "          m = j + 1;\n          break;",
     "          m = j + 2 < n ? j + 2 : n;\n          break;"),
    ("top-p compares strictly", "if (cum >= sel->p) {", "if (cum > sel->p) {"),
    ("threshold compares strictly", "for (int64_t i = 0; i < n; ++i) m += a[i] >= sel->tau;",
     "for (int64_t i = 0; i < n; ++i) m += a[i] > sel->tau;"),
    ("threshold may be empty", "      if (m < 1) m = 1;\n    } else {", "    } else {"),
    ("softmax of the rules unnormalised", "for (int64_t i = 0; i < n; ++i) a[i] /= z;", ""),
    ("block score is the block's last row", "for (int64_t i = 0; i < n; ++i) score[i / bs] += a[i];",
     "for (int64_t i = 0; i < n; ++i) score[i / bs] = a[i];"),
    ("short last block padded to full", "i < ((int64_t)blocks[j] + 1) * bs && i < n; ++i)",
     "i < ((int64_t)blocks[j] + 1) * bs; ++i)"),
    ("rule ignored in the step", "      ora_select(x, n, k, sel, Sout);", "      ora_topk(x, n, k, Sout);"),
    ("correction sees one row too few", "attend_rows(sh, qv, K, V, kv_base, NULL, p + 1, out + row * d, NULL);",
     "attend_rows(sh, qv, K, V, kv_base, NULL, p, out + row * d, NULL);"),
    ("correction without the causal mask", "const int64_t p = n - T + t;", "const int64_t p = n - 1;"),
    ("correction positions from the front", "const int64_t p = n - T + t;\n",
     "const int64_t p = t < n ? t : n - 1;\n"),
    ("correction reads the wrong KV group", "const int g = h / G;\n        const int64_t kv_base",
     "const int g = h % Hkv;\n        const int64_t kv_base"),
    ("smallest instead of largest", "if (a->x > b->x) return -1;\n  if (a->x < b->x) return 1;",
     "if (a->x < b->x) return -1;\n  if (a->x > b->x) return 1;"),
]


def caught(ora) -> str | None:
    for pin in P.ALL_PINS:
        try:
            pin(ora)
        except (AssertionError, ValueError) as e:   # a failed pin or a rejected call
            return f"{pin.__name__}: {str(e)[:80]}"
    return None


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = O.source_text()
    assert src.count(old) == 1, f"mutation anchor for '{name}' not unique in oracle.c"
    mutant = O.compile_variant(src.replace(old, new), str(tmp_path / "libmutant.so"))
    assert caught(mutant) is not None, f"no pin catches the planted mistake '{name}'"
