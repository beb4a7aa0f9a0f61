"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each pin takes an ``oracle.Oracle`` handle and raises AssertionError when the
oracle disagrees with a closed form, a textbook formula evaluated with numpy
or mpmath, a library sort, brute-force enumeration, or an invariant of the
method.  The same functions run against the real oracle
(test_oracle_pins.py) and against copies with planted mistakes
(test_oracle_mutants.py), which must each fail at least one pin.

Sources (page "LycheeDecode: Accelerating Long-Context LLM Inference via
Hybrid-Head Sparse Decoding", paper-graph-ui summary): section 3.4 Eq. (1)
dense retrieval attention, Eq. (2) argsTopK selection, Eq. (3) sparse
attention over the inherited set and the propagation rule that follows it,
the layer-0 initialisation, and the GQA pooling in the hyperparameter
summary.
"""
from __future__ import annotations

import itertools
import math

import mpmath
import numpy as np

import oracle as O

# ----------------------------------------------------------------- helpers


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (nearest even) and return the bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def widen(a: np.ndarray) -> np.ndarray:
    """Exact fp64 values of a uint16 (bf16) or float32 array."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def stack(q, k, v, role, mode=O.SELECT_PER_QHEAD) -> O.Stack:
    return O.Stack(np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v),
                   np.ascontiguousarray(role, dtype=np.uint8), mode)


def rand_stack(rng, L=2, B=1, Hq=4, Hkv=2, d=16, n=37, dtype="fp32", role=None,
               mode=O.SELECT_PER_QHEAD):
    q = rng.standard_normal((L, B, Hq, d))
    k = rng.standard_normal((L, B, Hkv, n, d))
    v = rng.standard_normal((L, B, Hkv, n, d))
    if role is None:
        role = np.zeros((L, Hq), dtype=np.uint8)
        role[0] = 1
    conv = bf16_bits if dtype == "bf16" else (lambda a: a.astype(np.float32))
    return stack(conv(q), conv(k), conv(v), role, mode)


def textbook_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """softmax(q K^T / sqrt(d)) V with numpy float64; also returns the logits."""
    d = q.shape[-1]
    logits = (K @ q) / np.sqrt(d)
    p = np.exp(logits - logits.max())
    p /= p.sum()
    return p @ V, logits


def library_topk(x: np.ndarray, k: int) -> np.ndarray:
    """numpy stable argsort of -x: larger first, equal values by lower index."""
    keff = min(k, x.size)
    sel = np.sort(np.argsort(-x, kind="stable")[:keff]).astype(np.int32)
    return np.concatenate([sel, np.full(k - keff, -1, dtype=np.int32)])


def close(a, b, atol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= atol, f"{what}: max abs error {err:.3e} > {atol:.1e}"


# ----------------------------------------------------------------- top-k pins


def pin_topk_distinct(ora):
    rng = np.random.default_rng(1)
    for n in (1, 2, 7, 100, 1000):
        x = rng.standard_normal(n)
        for k in sorted({1, 3, max(n - 1, 1), n, n + 5}):
            got = ora.topk(x, k)
            exp = library_topk(x, k)
            assert np.array_equal(got, exp), f"topk distinct n={n} k={k}: {got} vs {exp}"


def pin_topk_ties(ora):
    rng = np.random.default_rng(2)
    for n in (5, 64, 513):
        x = rng.integers(-2, 3, size=n).astype(np.float64)
        x[x == 0] = np.where(rng.random((x == 0).sum()) < 0.5, 0.0, -0.0)
        for k in (1, 2, n // 3 + 1, n - 1, n):
            got = ora.topk(x, k)
            exp = library_topk(x, k)
            assert np.array_equal(got, exp), f"topk ties n={n} k={k}"
    # all equal: the first k indices
    x = np.full(50, 1.25)
    assert np.array_equal(ora.topk(x, 7), np.arange(7, dtype=np.int32)), "all-equal keys"


def pin_topk_bruteforce(ora):
    """Enumerate every k-subset of tiny inputs: exactly one subset has every
    member ahead of every non-member (larger, or equal with a lower index)."""
    rng = np.random.default_rng(3)
    for trial in range(60):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, 5))
        x = rng.integers(-2, 3, size=n).astype(np.float64)
        keff = min(k, n)
        valid = []
        for T in itertools.combinations(range(n), keff):
            inside = set(T)
            ok = all(x[i] > x[j] or (x[i] == x[j] and i < j)
                     for i in inside for j in range(n) if j not in inside)
            if ok:
                valid.append(T)
        assert len(valid) == 1, f"brute force found {len(valid)} valid sets"
        exp = list(valid[0]) + [-1] * (k - keff)
        got = ora.topk(x, k)
        assert list(got) == exp, f"brute force n={n} k={k}: {list(got)} vs {exp}"


# ----------------------------------------------------------------- attention pins


def pin_closed_form_bf16(ora):
    """d=4, q=(2,0,0,0): logits = q.K/sqrt(4) = K[:,0] = (0, 1, 2); V rows are
    unit vectors, so o = (1, e, e^2, 0) / (1 + e + e^2).  All inputs are exact
    bf16 bit patterns (2.0 = 0x4000, 1.0 = 0x3F80)."""
    q = np.zeros((1, 1, 1, 4), dtype=np.uint16)
    q[0, 0, 0, 0] = 0x4000
    K = np.zeros((1, 1, 1, 3, 4), dtype=np.uint16)
    K[0, 0, 0, 1, 0] = 0x3F80
    K[0, 0, 0, 2, 0] = 0x4000
    V = np.zeros((1, 1, 1, 3, 4), dtype=np.uint16)
    for i in range(3):
        V[0, 0, 0, i, i] = 0x3F80
    st = stack(q, K, V, np.ones((1, 1)))
    out, S, _ = ora.decode_step(st, k=2)
    z = 1 + math.e + math.e ** 2
    close(out[0, 0, 0], [1 / z, math.e / z, math.e ** 2 / z, 0.0], 1e-15, "closed form")
    assert list(S[0, 0]) == [1, 2], f"closed-form top-2 {S[0, 0]}"


def pin_dense_textbook(ora):
    """Every head of layer 0: numpy softmax(qK^T/sqrt d)V, and S = library top-k."""
    rng = np.random.default_rng(4)
    for dtype in ("fp32", "bf16"):
        st = rand_stack(rng, L=1, B=2, Hq=6, Hkv=3, d=16, n=37, dtype=dtype)
        k = 9
        out, S, _ = ora.decode_step(st, k=k)
        G = 2
        for b in range(2):
            for h in range(6):
                g = h // G
                o, logits = textbook_attention(widen(st.q[0, b, h]), widen(st.k[0, b, g]),
                                               widen(st.v[0, b, g]))
                close(out[0, b, h], o, 1e-12, f"dense {dtype} b={b} h={h}")
                assert np.array_equal(S[b, h], library_topk(logits, k)), "dense selection"


def pin_mpmath_attention(ora):
    """Tiny case recomputed at 50 significant digits."""
    mpmath.mp.dps = 50
    rng = np.random.default_rng(5)
    st = rand_stack(rng, L=1, B=1, Hq=1, Hkv=1, d=3, n=5)
    out, _, _ = ora.decode_step(st, k=2)
    q = [mpmath.mpf(float(x)) for x in st.q[0, 0, 0]]
    K = st.k[0, 0, 0]
    V = st.v[0, 0, 0]
    s = [sum(q[j] * mpmath.mpf(float(K[i, j])) for j in range(3)) / mpmath.sqrt(3)
         for i in range(5)]
    w = [mpmath.e ** si for si in s]
    z = sum(w)
    exp = [float(sum(w[i] * mpmath.mpf(float(V[i, j])) for i in range(5)) / z) for j in range(3)]
    close(out[0, 0, 0], exp, 1e-14, "mpmath")


def pin_sparse_eq3(ora):
    """A sparse head attends over exactly its inherited rows, and passes the
    set on unchanged."""
    rng = np.random.default_rng(6)
    L, B, Hq, Hkv, d, n, k = 1, 2, 4, 2, 8, 40, 6
    role = np.array([[1, 0, 0, 1]], dtype=np.uint8)
    st = rand_stack(rng, L=L, B=B, Hq=Hq, Hkv=Hkv, d=d, n=n, role=role)
    S_in = np.stack([np.stack([np.sort(rng.choice(n, k, replace=False)) for _ in range(Hq)])
                     for _ in range(B)]).astype(np.int32)
    S_in[1, 2, 4:] = -1                # a shorter inherited set (padded)
    out, S_out, keys, fresh = ora.layer(st, 0, k, S_in, all_retrieval=False)
    assert list(fresh) == [1, 0, 0, 1], f"refreshed {fresh}"
    for b in range(B):
        for h in range(Hq):
            g = h // 2
            if role[0, h]:
                o, logits = textbook_attention(widen(st.q[0, b, h]), widen(st.k[0, b, g]),
                                               widen(st.v[0, b, g]))
                assert np.array_equal(S_out[b, h], library_topk(logits, k))
                close(keys[b, h], logits, 1e-13, "selection key = logits")
            else:
                rows = S_in[b, h][S_in[b, h] >= 0]
                o, _ = textbook_attention(widen(st.q[0, b, h]), widen(st.k[0, b, g][rows]),
                                          widen(st.v[0, b, g][rows]))
                assert np.array_equal(S_out[b, h], S_in[b, h]), "propagation"
            close(out[b, h], o, 1e-12, f"eq3 b={b} h={h}")


def pin_k_ge_n(ora):
    """k >= n: S is every row, and sparse heads equal dense heads bit for bit."""
    rng = np.random.default_rng(7)
    n = 23
    role_mixed = np.array([[1, 1, 1, 1], [1, 0, 0, 0]], dtype=np.uint8)
    st = rand_stack(rng, L=2, B=1, Hq=4, Hkv=2, d=8, n=n, role=role_mixed)
    st_dense = stack(st.q, st.k, st.v, np.ones((2, 4)))
    for k in (n, n + 4):
        out_m, S_m, _ = ora.decode_step(st, k=k)
        out_d, S_d, _ = ora.decode_step(st_dense, k=k)
        assert np.array_equal(out_m, out_d), "sparse != dense at k >= n"
        exp = np.concatenate([np.arange(n), np.full(k - n, -1)]).astype(np.int32)
        for h in range(4):
            assert np.array_equal(S_m[0, h], exp), "k >= n selection"


def pin_uniform_keys(ora):
    """All keys equal: every weight is 1/n, so o = mean(V); ties select 0..k-1."""
    rng = np.random.default_rng(8)
    st = rand_stack(rng, L=2, B=1, Hq=4, Hkv=2, d=8, n=50,
                    role=np.array([[1, 1, 1, 1], [0, 1, 0, 0]]))
    st.k[:] = st.k[:, :, :, :1, :]
    k = 11
    out, S, tr = ora.decode_step(st, k=k, trace=True)
    for h in range(4):
        close(out[0, 0, h], widen(st.v[0, 0, h // 2]).mean(axis=0), 1e-14, "uniform keys")
        # layer 1: the retrieval head averages every row, sparse heads their set
        rows = slice(None) if h == 1 else tr[0, 0, h]
        close(out[1, 0, h], widen(st.v[1, 0, h // 2])[rows].mean(axis=0), 1e-14,
              "uniform keys, layer 1")
    for h in range(4):
        assert np.array_equal(tr[0, 0, h], np.arange(k)), "uniform-key tie break"


def pin_planted_key(ora):
    """A key planted as c * q_h (c large) is always in that head's set."""
    rng = np.random.default_rng(9)
    st = rand_stack(rng, L=1, B=1, Hq=4, Hkv=2, d=16, n=200)
    plant = {0: 17, 1: 160, 2: 5, 3: 99}
    for h, j in plant.items():
        st.k[0, 0, h // 2, j] = (6.0 * st.q[0, 0, h]).astype(np.float32)
    _, S, _ = ora.decode_step(st, k=8)
    for h, j in plant.items():
        assert j in set(S[0, h].tolist()), f"planted key {j} missing for head {h}"


def pin_chain(ora):
    """Sparse heads pass the set on unchanged, layer after layer; a retrieval
    head replaces it.  Layer 3's sparse head attends over layer 0's set."""
    rng = np.random.default_rng(10)
    L = 5
    role = np.zeros((L, 4), dtype=np.uint8)
    role[0] = 1
    role[2, 1] = 1
    st = rand_stack(rng, L=L, B=1, Hq=4, Hkv=2, d=8, n=60, role=role)
    k = 7
    out, S, tr = ora.decode_step(st, k=k, trace=True)
    for l in range(1, L):
        assert np.array_equal(tr[l, 0, 0], tr[0, 0, 0]), "head 0 chain"
    assert np.array_equal(tr[1, 0, 1], tr[0, 0, 1])
    assert not np.array_equal(tr[2, 0, 1], tr[1, 0, 1]), "refresh at layer 2 expected"
    for l in (3, 4):
        assert np.array_equal(tr[l, 0, 1], tr[2, 0, 1]), "head 1 chain after refresh"
    assert np.array_equal(S, tr[L - 1]), "final S = last trace entry"
    rows = tr[0, 0, 0]
    o, _ = textbook_attention(widen(st.q[3, 0, 0]), widen(st.k[3, 0, 0][rows]),
                              widen(st.v[3, 0, 0][rows]))
    close(out[3, 0, 0], o, 1e-12, "layer-3 sparse head over layer-0 set")
    # the layer-2 selection of head 1 is the top-k of its own layer-2 logits
    _, logits = textbook_attention(widen(st.q[2, 0, 1]), widen(st.k[2, 0, 0]), widen(st.v[2, 0, 0]))
    assert np.array_equal(tr[2, 0, 1], library_topk(logits, k)), "layer-2 refresh"


def pin_layer0_forced(ora):
    """Role row 0 is ignored when no set is given: layer 0 is all retrieval."""
    rng = np.random.default_rng(11)
    st = rand_stack(rng, L=2, B=1, Hq=4, Hkv=2, d=8, n=30,
                    role=np.array([[0, 0, 0, 0], [0, 1, 0, 0]]))
    st1 = stack(st.q, st.k, st.v, np.array([[1, 1, 1, 1], [0, 1, 0, 0]]))
    a = ora.decode_step(st, k=5)
    b = ora.decode_step(st1, k=5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]), "layer-0 rule"


def pin_permutation(ora):
    """Permuting the cache rows leaves every output unchanged and maps S."""
    rng = np.random.default_rng(12)
    n = 48
    role = np.array([[1, 1, 1, 1], [1, 0, 0, 0]], dtype=np.uint8)
    st = rand_stack(rng, L=2, B=1, Hq=4, Hkv=2, d=8, n=n, role=role)
    perm = rng.permutation(n)          # new row i holds old token perm[i]
    stp = stack(st.q, st.k[:, :, :, perm], st.v[:, :, :, perm], role)
    k = 9
    out, S, tr = ora.decode_step(st, k=k, trace=True)
    outp, Sp, trp = ora.decode_step(stp, k=k, trace=True)
    close(out, outp, 1e-12, "permutation outputs")
    for l in range(2):
        for h in range(4):
            assert set(perm[trp[l, 0, h]].tolist()) == set(tr[l, 0, h].tolist()), "mapped S"


def pin_linearity(ora):
    """o is linear in V (exact fp32 inputs), constant V gives constant o, and
    k = 1 selects the argmax."""
    rng = np.random.default_rng(13)
    base = rand_stack(rng, L=1, B=1, Hq=4, Hkv=2, d=8, n=33)
    V1 = rng.integers(-4, 5, size=base.v.shape).astype(np.float32)
    V2 = rng.integers(-4, 5, size=base.v.shape).astype(np.float32)
    V3 = (2 * V1 - 3 * V2).astype(np.float32)
    o1 = ora.decode_step(stack(base.q, base.k, V1, base.role), k=3)[0]
    o2 = ora.decode_step(stack(base.q, base.k, V2, base.role), k=3)[0]
    o3 = ora.decode_step(stack(base.q, base.k, V3, base.role), k=3)[0]
    close(o3, 2 * o1 - 3 * o2, 1e-12, "linearity in V")
    Vc = np.full(base.v.shape, 0.375, dtype=np.float32)
    oc = ora.decode_step(stack(base.q, base.k, Vc, base.role), k=3)[0]
    close(oc, np.full(oc.shape, 0.375), 1e-15, "constant V")
    _, S1, _ = ora.decode_step(base, k=1)
    for h in range(4):
        logits = widen(base.k[0, 0, h // 2]) @ widen(base.q[0, 0, h])
        assert S1[0, h, 0] == int(np.argmax(logits)), "k=1 is argmax"


def pin_kvgroup(ora):
    """Group mode: the selection key is the mean-pooled query's logit, one set
    per KV group, shared by every sparse head of the group."""
    rng = np.random.default_rng(14)
    L, B, Hq, Hkv, d, n, k = 2, 2, 6, 2, 8, 45, 7
    G = Hq // Hkv
    role = np.zeros((L, Hq), dtype=np.uint8)
    role[0] = 1
    role[1, 4] = 1                     # group 1 refreshed at layer 1, group 0 not
    st = rand_stack(rng, L=L, B=B, Hq=Hq, Hkv=Hkv, d=d, n=n, role=role,
                    mode=O.SELECT_KVGROUP_MEAN)
    out, S, tr = ora.decode_step(st, k=k, trace=True)
    assert tr.shape == (L, B, Hkv, k)
    for b in range(B):
        for g in range(Hkv):
            qbar = widen(st.q[0, b, g * G:(g + 1) * G]).mean(axis=0)
            logits = widen(st.k[0, b, g]) @ qbar / np.sqrt(d)
            assert np.array_equal(tr[0, b, g], library_topk(logits, k)), "group key"
        # layer 1: group 0 keeps its set; heads 0-2 attend over it
        assert np.array_equal(tr[1, b, 0], tr[0, b, 0])
        rows = tr[0, b, 0]
        for h in range(G):
            o, _ = textbook_attention(widen(st.q[1, b, h]), widen(st.k[1, b, 0][rows]),
                                      widen(st.v[1, b, 0][rows]))
            close(out[1, b, h], o, 1e-12, "group sparse head")
        # group 1 is refreshed from layer 1's pooled query; its sparse heads
        # (3 and 5) still attend over the set they inherited
        qbar = widen(st.q[1, b, G:2 * G]).mean(axis=0)
        logits = widen(st.k[1, b, 1]) @ qbar / np.sqrt(d)
        assert np.array_equal(tr[1, b, 1], library_topk(logits, k)), "group refresh"
        rows = tr[0, b, 1]
        for h in (3, 5):
            o, _ = textbook_attention(widen(st.q[1, b, h]), widen(st.k[1, b, 1][rows]),
                                      widen(st.v[1, b, 1][rows]))
            close(out[1, b, h], o, 1e-12, "group sparse head, refreshed group")
        o, _ = textbook_attention(widen(st.q[1, b, 4]), widen(st.k[1, b, 1]), widen(st.v[1, b, 1]))
        close(out[1, b, 4], o, 1e-12, "group retrieval head")


def pin_strided_layout(ora):
    """The oracle reads the cache through its strides: a cache allocated with
    more rows than n gives the same result as the exact-size cache."""
    rng = np.random.default_rng(15)
    big = rand_stack(rng, L=2, B=2, Hq=4, Hkv=2, d=8, n=40,
                     role=np.array([[1, 1, 1, 1], [0, 0, 1, 0]]))
    n = 29
    small = stack(big.q, big.k[:, :, :, :n].copy(), big.v[:, :, :, :n].copy(), big.role)
    a = ora.decode_step(big, k=6, n=n)
    b = ora.decode_step(small, k=6)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]), "strided cache"
    # rows padded past d with junk: the token stride is the padded row
    pad = np.full(small.k.shape[:-1] + (5,), 7.0, dtype=np.float32)
    padded = stack(small.q, np.concatenate([small.k, pad], axis=-1),
                   np.concatenate([small.v, -pad], axis=-1), small.role)
    c = ora.decode_step(padded, k=6)
    assert np.array_equal(c[0], b[0]) and np.array_equal(c[1], b[1]), "padded rows"


def pin_batch_elements_independent(ora):
    """Batch elements do not interact (sets are per element; Algorithm 1 runs
    per sequence), which is what lets the serving form check each element of a
    variable-length batch as a one-element step over its own rows: the
    batched oracle equals its per-element runs, and an element's results do
    not move when another element's cache changes."""
    rng = np.random.default_rng(16)
    role = np.array([[1, 1, 1, 1], [0, 1, 0, 0], [1, 0, 0, 1]], dtype=np.uint8)
    st = rand_stack(rng, L=3, B=3, Hq=4, Hkv=2, d=8, n=33, role=role)
    out, S, _ = ora.decode_step(st, k=5)
    for b in range(3):
        one = stack(st.q[:, b:b + 1].copy(), st.k[:, b:b + 1].copy(), st.v[:, b:b + 1].copy(), role)
        o1, S1, _ = ora.decode_step(one, k=5)
        assert np.array_equal(o1[:, 0], out[:, b]) and np.array_equal(S1[0], S[b]), f"element {b}"
    k2 = st.k.copy()
    k2[:, 1] = rng.standard_normal(k2[:, 1].shape).astype(np.float32)
    out2, S2, _ = ora.decode_step(stack(st.q, k2, st.v, role), k=5)
    assert np.array_equal(out2[:, 0], out[:, 0]) and np.array_equal(out2[:, 2], out[:, 2])
    assert np.array_equal(S2[0], S[0]) and np.array_equal(S2[2], S[2])
    assert not np.array_equal(out2[:, 1], out[:, 1]), "element 1 must see its own change"


# ----------------------------------------------------------------- selection rules
# Section 4.4.1 (Figure 6, Tables 5-6) names the rules; the readings (set sizes,
# order, the cap k, blocks scored by summed probability) are the oracle's.


def softmax64(x: np.ndarray) -> np.ndarray:
    e = np.exp(x - x.max())
    return e / e.sum()


def padded(rows, k):
    rows = list(rows)
    return np.array(rows + [-1] * (k - len(rows)), dtype=np.int32)


def pin_select_topk_rule_is_topk(ora):
    rng = np.random.default_rng(40)
    x = rng.standard_normal(77)
    for k in (1, 9, 77, 90):
        assert np.array_equal(ora.select(x, k, O.Selection(O.RULE_TOPK)), library_topk(x, k))


def pin_select_ratio(ora):
    """ceil(num/den * n) rows (integer arithmetic), at least 1, at most k; the
    reasoning budget (ratio 1/2) grows by one row every two steps."""
    rng = np.random.default_rng(41)
    for n in (1, 7, 10, 64, 301):
        x = rng.standard_normal(n)
        for num, den in ((1, 2), (7, 10), (1, 3), (0, 1), (3, 2), (1, 1000)):
            m = max(1, -((-num * n) // den))
            for k in (1, 5, 200, 400):
                exp = library_topk(x, min(m, k))
                exp = np.concatenate([exp, np.full(k - exp.size, -1, dtype=np.int32)])
                got = ora.select(x, k, O.Selection(O.RULE_RATIO, ratio=(num, den)))
                assert np.array_equal(got, exp), f"ratio {num}/{den} n={n} k={k}"
    x = rng.standard_normal(40)
    sizes = [int((ora.select(x[:n], 64, O.Selection(O.RULE_RATIO, ratio=(1, 2))) >= 0).sum())
             for n in range(1, 41)]
    assert sizes == [(n + 1) // 2 for n in range(1, 41)], sizes


def pin_select_topp(ora):
    """Known probabilities (1/2, 1/4, 1/8, 1/8), uniform keys, the cap, and
    brute force: no smaller subset reaches the mass p, and the greedy set is
    the top-m by key."""
    w = np.array([0.125, 0.5, 0.125, 0.25])
    x = np.log(w)
    for pv, exp in ((0.3, [1]), (0.6, [1, 3]), (0.74, [1, 3]), (0.76, [0, 1, 3]),
                    (0.87, [0, 1, 3]), (0.88, [0, 1, 2, 3]), (1.0, [0, 1, 2, 3])):
        got = ora.select(x, 6, O.Selection(O.RULE_TOPP, p=pv))
        assert np.array_equal(got, padded(exp, 6)), f"top-p {pv}: {got}"
    assert np.array_equal(ora.select(x, 2, O.Selection(O.RULE_TOPP, p=0.99)), padded([1, 3], 2))
    # uniform keys: A = 1/n, ties by index, m = ceil(p n)
    for n in (8, 13):
        for j in range(n):
            pv = (j + 0.5) / n
            got = ora.select(np.zeros(n), n, O.Selection(O.RULE_TOPP, p=pv))
            assert np.array_equal(got, padded(range(j + 1), n)), f"uniform top-p n={n} j={j}"
    # mass reached exactly (n = 8: A = 1/8 and every running sum are exact):
    # the row that reaches p is the last one taken
    for j in range(8):
        got = ora.select(np.zeros(8), 8, O.Selection(O.RULE_TOPP, p=(j + 1) / 8))
        assert np.array_equal(got, padded(range(j + 1), 8)), f"exact mass {j + 1}/8"
    rng = np.random.default_rng(42)
    for trial in range(80):
        n = int(rng.integers(1, 9))
        x = rng.standard_normal(n) * 2.0
        a = softmax64(x)
        pv = float(rng.uniform(0.05, 0.99))
        got = ora.select(x, n, O.Selection(O.RULE_TOPP, p=pv))
        m = int((got >= 0).sum())
        best = min(len(T) for r in range(1, n + 1) for T in itertools.combinations(range(n), r)
                   if a[list(T)].sum() >= pv - 1e-12)
        assert m == best, f"top-p brute force: {m} vs {best}"
        assert np.array_equal(got, padded(library_topk(x, m), n)), "top-p set is not the top-m"


def pin_select_threshold(ora):
    """Rows with A >= tau: exact probabilities (uniform over 8 rows gives
    A = 1/8 exactly), at least one row, at most k; numpy count elsewhere."""
    assert np.array_equal(ora.select(np.zeros(8), 8, O.Selection(O.RULE_THRESHOLD, tau=0.125)),
                          np.arange(8, dtype=np.int32))
    assert np.array_equal(ora.select(np.zeros(8), 8, O.Selection(O.RULE_THRESHOLD, tau=0.13)),
                          padded([0], 8))
    x = np.log(np.array([0.125, 0.5, 0.125, 0.25]))
    assert np.array_equal(ora.select(x, 4, O.Selection(O.RULE_THRESHOLD, tau=0.2)), padded([1, 3], 4))
    assert np.array_equal(ora.select(x, 4, O.Selection(O.RULE_THRESHOLD, tau=0.9)), padded([1], 4))
    rng = np.random.default_rng(43)
    for trial in range(40):
        n = int(rng.integers(1, 300))
        x = rng.standard_normal(n) * 3.0
        a = softmax64(x)
        tau = float(10 ** rng.uniform(-4, -0.5))
        k = int(rng.integers(1, 400))
        m = min(max(1, int((a >= tau).sum())), k, n)
        got = ora.select(x, k, O.Selection(O.RULE_THRESHOLD, tau=tau))
        assert np.array_equal(got, np.concatenate([library_topk(x, m),
                                                   np.full(k - m, -1, dtype=np.int32)]))


def pin_select_block(ora):
    """Block 1 is top-k; blocks scored by summed probability (numpy), the
    floor(k/block) best taken whole (ties to the lower block), the short last
    block included; planted keys pick their blocks."""
    rng = np.random.default_rng(44)
    x = rng.standard_normal(50)
    for k in (1, 7, 50, 60):
        assert np.array_equal(ora.select(x, k, O.Selection(O.RULE_BLOCK_TOPK, block=1)),
                              library_topk(x, k))
    for trial in range(40):
        n = int(rng.integers(1, 400))
        bs = int(rng.choice([2, 4, 16, 64]))
        k = int(rng.integers(bs, 6 * bs + 1))
        x = rng.standard_normal(n) * 2.0
        starts = np.arange(0, n, bs)
        score = np.add.reduceat(softmax64(x), starts)
        kb = min(k // bs, starts.size)
        blocks = np.sort(np.argsort(-score, kind="stable")[:kb])
        rows = [i for b in blocks for i in range(b * bs, min(n, (b + 1) * bs))]
        got = ora.select(x, k, O.Selection(O.RULE_BLOCK_TOPK, block=bs))
        assert np.array_equal(got, padded(rows, k)), f"block n={n} bs={bs} k={k}"
    x = np.zeros(10)
    x[9] = 8.0
    assert np.array_equal(ora.select(x, 4, O.Selection(O.RULE_BLOCK_TOPK, block=4)), padded([8, 9], 4))
    x = np.zeros(12)   # equal blocks: the lowest ones
    assert np.array_equal(ora.select(x, 8, O.Selection(O.RULE_BLOCK_TOPK, block=4)),
                          np.arange(8, dtype=np.int32))
    with np.testing.assert_raises(ValueError):
        ora.select(x, 3, O.Selection(O.RULE_BLOCK_TOPK, block=4))   # k below one block


def pin_select_in_step(ora):
    """Through a whole step: every refreshed set is the rule applied to the
    layer's keys (the head's logits), and a sparse head attends over exactly
    the rows of its variable-size set (textbook attention over them)."""
    rng = np.random.default_rng(45)
    role = np.array([[1, 1], [0, 1], [0, 0]], dtype=np.uint8)
    st = rand_stack(rng, L=3, B=1, Hq=2, Hkv=1, d=8, n=40, role=role)
    q, K, V = widen(st.q), widen(st.k), widen(st.v)
    for sel in (O.Selection(O.RULE_TOPP, p=0.5), O.Selection(O.RULE_THRESHOLD, tau=0.03),
                O.Selection(O.RULE_RATIO, ratio=(1, 4)), O.Selection(O.RULE_BLOCK_TOPK, block=4)):
        out, S, tr = ora.decode_step(st, k=16, trace=True, sel=sel)
        for l in range(3):
            for h in range(2):
                if l == 0 or role[l, h]:
                    _, logits = textbook_attention(q[l, 0, h], K[l, 0, 0], V[l, 0, 0])
                    exp = ora.select(logits, 16, sel)
                    assert np.array_equal(tr[l, 0, h], exp), f"rule {sel.rule} l={l} h={h}"
                else:
                    rows = tr[l - 1, 0, h]
                    rows = rows[rows >= 0]
                    o, _ = textbook_attention(q[l, 0, h], K[l, 0, 0][rows], V[l, 0, 0][rows])
                    close(out[l, 0, h], o, 1e-12, f"sparse head over a rule-{sel.rule} set")
                    assert np.array_equal(tr[l, 0, h], tr[l - 1, 0, h])


# ----------------------------------------------------------------- cache correction
# Section 4.2.2: every 32 decoded tokens the T most recent positions are
# prefilled again with dense attention; query t sits at position n - T + t.


def pin_correction_textbook_causal(ora):
    """numpy causal attention over a random cache, fp32 and bf16: query t of
    every head attends rows 0 .. n - T + t."""
    rng = np.random.default_rng(50)
    for dtype, n, T in (("fp32", 23, 5), ("bf16", 40, 8), ("fp32", 6, 6)):
        st = rand_stack(rng, L=2, B=2, Hq=4, Hkv=2, d=8, n=n, dtype=dtype)
        qf = rng.standard_normal((2, 2, 4, T, 8))
        q = bf16_bits(qf) if dtype == "bf16" else qf.astype(np.float32)
        got = ora.correction(st, q)
        Q, K, V = widen(q), widen(st.k), widen(st.v)
        for l in range(2):
            for b in range(2):
                for h in range(4):
                    g = h // 2
                    for t in range(T):
                        p = n - T + t
                        o, _ = textbook_attention(Q[l, b, h, t], K[l, b, g, :p + 1], V[l, b, g, :p + 1])
                        close(got[l, b, h, t], o, 1e-12, f"correction {dtype} l{l} b{b} h{h} t{t}")


def pin_correction_causality(ora):
    """Changing cache row r moves exactly the queries at positions >= r."""
    rng = np.random.default_rng(51)
    n, T = 30, 6
    st = rand_stack(rng, L=1, B=1, Hq=2, Hkv=1, d=8, n=n)
    q = rng.standard_normal((1, 1, 2, T, 8)).astype(np.float32)
    base = ora.correction(st, q)
    for r in (n - T, n - 3, n - 1):
        k2, v2 = st.k.copy(), st.v.copy()
        k2[0, 0, 0, r] += 1.0
        v2[0, 0, 0, r] -= 2.0
        moved = ora.correction(stack(st.q, k2, v2, st.role), q)
        for t in range(T):
            same = np.array_equal(moved[0, 0, :, t], base[0, 0, :, t])
            assert same == (n - T + t < r), f"row {r} query {t}: causality broken"


def pin_correction_last_query_is_decode(ora):
    """The last query (position n - 1) is the decode step's dense attention
    of a retrieval head over all n rows (Eq. 1, layer 0 all retrieval)."""
    rng = np.random.default_rng(52)
    n, T = 33, 4
    st = rand_stack(rng, L=1, B=2, Hq=4, Hkv=2, d=16, n=n)
    q = rng.standard_normal((1, 2, 4, T, 16)).astype(np.float32)
    got = ora.correction(st, q)
    last = stack(np.ascontiguousarray(q[:, :, :, T - 1]), st.k, st.v, st.role)
    out, _, _, _ = ora.layer(last, 0, 4, None, all_retrieval=True)
    close(got[0, :, :, T - 1], out, 1e-13, "last correction query vs the dense decode pass")


ALL_PINS = [
    pin_topk_distinct, pin_topk_ties, pin_topk_bruteforce, pin_closed_form_bf16,
    pin_dense_textbook, pin_mpmath_attention, pin_sparse_eq3, pin_k_ge_n, pin_uniform_keys,
    pin_planted_key, pin_chain, pin_layer0_forced, pin_permutation, pin_linearity,
    pin_kvgroup, pin_strided_layout, pin_batch_elements_independent,
    pin_select_topk_rule_is_topk, pin_select_ratio, pin_select_topp, pin_select_threshold,
    pin_select_block, pin_select_in_step, pin_correction_textbook_causal,
    pin_correction_causality, pin_correction_last_query_is_decode,
]
