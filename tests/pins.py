"""Pins for the fp64 oracle: facts fixed by the pages or by mathematics.

Each pin takes an `oracle.Oracle` and raises AssertionError when the oracle
disagrees with something that does not come from the oracle itself:
  - hand-worked examples (tests/golden/hand_examples.txt);
  - the R = 0 identity with softmax attention, checked against torch's own
    softmax and matmul ("Integrazioni AI personalizzate dopo l'attenzione
    Parallax", encorp.ai, FAQ: zero projection gives softmax attention);
  - the local-linear reading: with the probe set to the LLA solver output
    Sigma_w^{-1}(q - kbar), the output equals the intercept of the weighted
    least-squares line, solved here by numpy's lstsq ("Parallax: Parameterized
    Local Linear Attention for Language Modeling", bayesiansapien blog,
    opening diagram: LLA is the local linear estimate);
  - closed forms, invariances and brute-force agreement between the forms.

test_oracle_pins.py runs them on the real oracle; test_oracle_mutants.py
checks that each planted mistake in a copy of the oracle trips one of them.
"""
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

FORMS = ("covariance", "expanded", "streaming3", "streaming1")


def run_form(orc, form, q, r, k, v, n, scale):
    if form == "covariance":
        return orc.parallax_covariance(q, r, k, v, n, scale)
    if form == "expanded":
        return orc.parallax_expanded(q, r, k, v, n, scale)
    if form == "streaming3":
        return orc.parallax_streaming(q, r, k, v, n, scale, 3)
    if form == "streaming1":
        return orc.parallax_streaming(q, r, k, v, n, scale, 1)
    raise ValueError(form)


def all_forms(orc, q, r, k, v, n, scale):
    return {f: run_form(orc, f, q, r, k, v, n, scale) for f in FORMS}


def rand_case(seed, B=2, Hq=4, Hkv=2, D=8, Lmax=24, lengths=(11, 24), r_scale=0.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, D))
    r = rng.standard_normal((B, Hq, D)) * r_scale
    k = rng.standard_normal((B, Hkv, Lmax, D))
    v = rng.standard_normal((B, Hkv, Lmax, D))
    n = np.array(lengths, dtype=np.int32)
    return q, r, k, v, n


def close(a, b, tol=1e-11, what=""):
    a, b = np.asarray(a), np.asarray(b)
    err = np.max(np.abs(a - b) / np.maximum(1.0, np.abs(b))) if a.size else 0.0
    assert np.all(np.isfinite(a)), f"{what}: non-finite output"
    assert err <= tol, f"{what}: max scaled error {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- golden ----

def load_hand_examples():
    examples, cur = [], None
    with open(os.path.join(GOLDEN, "hand_examples.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (x.strip() for x in line.split("=", 1))
            if key == "name":
                cur = {"name": val, "k": [], "v": []}
                examples.append(cur)
            elif key in ("k", "v"):
                cur[key].append([float(x) for x in val.split()])
            elif key == "scale":
                cur[key] = float(val)
            else:
                cur[key] = [float(x) for x in val.split()]
    return examples


def pin_hand_examples(orc):
    for ex in load_hand_examples():
        n = len(ex["k"])
        q = np.array(ex["q"])[None, None, :]
        r = np.array(ex["r"])[None, None, :]
        k = np.array(ex["k"])[None, None, :, :]
        v = np.array(ex["v"])[None, None, :, :]
        want = np.array(ex["o"])[None, None, :]
        for form, got in all_forms(orc, q, r, k, v, [n], ex["scale"]).items():
            close(got, want, 1e-12, f"{ex['name']} ({form})")
        if not np.any(r):
            close(orc.softmax_decode(q, k, v, [n], ex["scale"]), want, 1e-12,
                  f"{ex['name']} (softmax)")


# ------------------------------------------------------ R = 0 is softmax ----

def torch_softmax_attention(q, k, v, n, scale):
    """softmax(scale q K^T) V per head with torch's own routines (fp64)."""
    q, k, v = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    B, Hq, D = q.shape
    G = Hq // k.shape[1]
    kk = torch.repeat_interleave(k, G, dim=1)  # [B, Hq, Lmax, D]
    vv = torch.repeat_interleave(v, G, dim=1)
    out = torch.zeros(B, Hq, D, dtype=torch.float64)
    for b in range(B):
        nb = int(n[b])
        if nb == 0:
            continue
        logits = scale * torch.einsum("hd,hld->hl", q[b], kk[b, :, :nb])
        out[b] = torch.einsum("hl,hld->hd", torch.softmax(logits, dim=-1), vv[b, :, :nb])
    return out.numpy()


def pin_r_zero_is_softmax(orc):
    q, r, k, v, n = rand_case(1, B=3, Hq=6, Hkv=2, D=16, Lmax=40, lengths=(17, 40, 1))
    want = torch_softmax_attention(q, k, v, n, 0.25)
    zero = np.zeros_like(r)
    for form, got in all_forms(orc, q, zero, k, v, n, 0.25).items():
        close(got, want, 1e-12, f"r=0 ({form})")
    close(orc.softmax_decode(q, k, v, n, 0.25), want, 1e-12, "softmax_decode")


# ---------------------------------------------------------- closed forms ----

def pin_single_key_returns_v(orc):
    q, r, k, v, _ = rand_case(2, lengths=(1, 1))
    want = np.repeat(v[:, :, 0, :], 2, axis=1)  # G = 2
    for form, got in all_forms(orc, q, r, k, v, [1, 1], 0.3).items():
        close(got, want, 1e-12, f"single key ({form})")


def pin_constant_values(orc):
    q, r, k, v, n = rand_case(3)
    c = np.random.default_rng(30).standard_normal((2, 2, 1, 8))
    v = np.broadcast_to(c, v.shape).copy()
    want = np.repeat(c[:, :, 0, :], 2, axis=1)
    for form, got in all_forms(orc, q, r, k, v, n, 0.3).items():
        close(got, want, 1e-12, f"constant V ({form})")


def pin_value_shift_and_scale(orc):
    q, r, k, v, n = rand_case(4)
    base = orc.parallax_covariance(q, r, k, v, n, 0.3)
    c = np.random.default_rng(40).standard_normal(8)
    for form in FORMS:
        close(run_form(orc, form, q, r, k, v + c, n, 0.3), base + c, 1e-11,
              f"V + c ({form})")
        close(run_form(orc, form, q, r, k, -2.5 * v, n, 0.3), -2.5 * base, 1e-11,
              f"alpha V ({form})")


# ------------------------------------------------------------ invariants ----

def pin_key_translation(orc):
    """k_i -> k_i + u adds q.u to every logit and r.u to every probe score;
    neither changes o. A large u also exercises the max subtraction."""
    q, r, k, v, n = rand_case(5)
    base = orc.parallax_covariance(q, r, k, v, n, 0.3)
    u = 40.0 * np.random.default_rng(50).standard_normal(8)
    for form in FORMS:
        close(run_form(orc, form, q, r, k + u, v, n, 0.3), base, 1e-9,
              f"k + u ({form})")


def pin_linear_in_r(orc):
    q, r1, k, v, n = rand_case(6)
    r2 = np.random.default_rng(60).standard_normal(r1.shape)
    for form in FORMS:
        f = lambda r: run_form(orc, form, q, r, k, v, n, 0.3)
        o0, o1, o2 = f(np.zeros_like(r1)), f(r1), f(r2)
        close(f(r1 + r2) - o0, (o1 - o0) + (o2 - o0), 1e-10, f"additive in r ({form})")
        close(f(-3.0 * r1) - o0, -3.0 * (o1 - o0), 1e-10, f"homogeneous in r ({form})")
        # the correction is not identically zero
        assert np.max(np.abs(o1 - o0)) > 1e-3, f"r has no effect ({form})"


def pin_key_permutation(orc):
    q, r, k, v, n = rand_case(7, lengths=(24, 24))
    perm = np.random.default_rng(70).permutation(24)
    base = orc.parallax_covariance(q, r, k, v, n, 0.3)
    for form in FORMS:
        close(run_form(orc, form, q, r, k[:, :, perm], v[:, :, perm], n, 0.3), base,
              1e-11, f"key permutation ({form})")


def pin_forms_agree(orc):
    """Brute force: definition, expansion and chunked streaming agree."""
    q, r, k, v, n = rand_case(8, B=4, Hq=8, Hkv=2, D=16, Lmax=70, lengths=(70, 1, 33, 64))
    base = orc.parallax_covariance(q, r, k, v, n, 0.25)
    close(orc.parallax_expanded(q, r, k, v, n, 0.25), base, 1e-11, "expanded")
    for chunk in (1, 2, 5, 16, 64, 70, 1000):
        close(orc.parallax_streaming(q, r, k, v, n, 0.25, chunk), base, 1e-11,
              f"streaming chunk={chunk}")


# ------------------------------------------- local linear (LLA) intercept ----

def pin_local_linear_intercept(orc):
    """With r = Sigma_w^{-1}(q - kbar) (LLA's solver output) the Parallax
    output is the intercept at q of the weighted least-squares fit
    v_i ~ a + M (k_i - q), weights w_i = softmax(scale q.k_i)."""
    rng = np.random.default_rng(9)
    D, n, scale = 4, 15, 0.7
    q = rng.standard_normal(D)
    k = rng.standard_normal((n, D))
    v = rng.standard_normal((n, D))
    t = scale * k @ q
    w = np.exp(t - t.max())
    w /= w.sum()
    kbar = w @ k
    sigma = (k - kbar).T @ ((k - kbar) * w[:, None])
    r = np.linalg.solve(sigma, q - kbar)
    # weighted least squares with an intercept column
    X = np.hstack([np.ones((n, 1)), k - q])
    sw = np.sqrt(w)[:, None]
    coef, *_ = np.linalg.lstsq(X * sw, v * sw, rcond=None)
    intercept = coef[0]
    for form, got in all_forms(orc, q[None, None], r[None, None], k[None, None],
                               v[None, None], [n], scale).items():
        close(got[0, 0], intercept, 1e-9, f"LLA intercept ({form})")


# ----------------------------------------------- layout, GQA and lengths ----

def pin_gqa_mapping(orc):
    """Query head h reads kv head h // (Hq/Hkv): give kv head g values g+1."""
    for Hq, Hkv in ((8, 2), (8, 8), (8, 1), (12, 3)):
        q, r, k, v, n = rand_case(10, Hq=Hq, Hkv=Hkv)
        v = np.zeros_like(v)
        for g in range(Hkv):
            v[:, g] = g + 1.0
        want = np.zeros((2, Hq, 8))
        for h in range(Hq):
            want[:, h, :] = h // (Hq // Hkv) + 1.0
        for form, got in all_forms(orc, q, r, k, v, n, 0.3).items():
            close(got, want, 1e-12, f"GQA {Hq}/{Hkv} ({form})")


def pin_lengths_exact(orc):
    """q = 0 (equal weights), r = 0, value of key i = i: o = (n-1)/2 exactly
    when exactly keys 0..n-1 are read. NaN padding must not leak."""
    lengths = (1, 2, 7, 24)
    q, r, k, v, n = rand_case(11, B=4, lengths=lengths)
    q[:] = 0.0
    r[:] = 0.0
    for i in range(24):
        v[:, :, i, :] = float(i)
    for b, nb in enumerate(lengths):
        k[b, :, nb:, :] = np.nan
        v[b, :, nb:, :] = np.nan
    want = np.zeros((4, 4, 8))
    for b, nb in enumerate(lengths):
        want[b] = (nb - 1) / 2.0
    for form, got in all_forms(orc, q, r, k, v, n, 0.3).items():
        close(got, want, 1e-12, f"lengths ({form})")
    close(orc.softmax_decode(q, k, v, n, 0.3), want, 1e-12, "lengths (softmax)")


def pin_empty_sequence_is_zero(orc):
    q, r, k, v, _ = rand_case(12)
    n = [0, 5]
    k[0] = np.nan
    v[0] = np.nan
    for form, got in all_forms(orc, q, r, k, v, n, 0.3).items():
        assert np.all(got[0] == 0.0), f"empty sequence ({form})"
        assert np.all(np.isfinite(got[1])), f"finite ({form})"


# ------------------------------------------------------------------ prefill --

def rand_prefill(seed, B=2, Hq=4, Hkv=2, L=12, D=8, r_scale=0.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, L, D))
    r = rng.standard_normal((B, Hq, L, D)) * r_scale
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    return q, r, k, v


def torch_sdpa(q, k, v, scale, causal):
    """torch's own scaled_dot_product_attention in fp64 (GQA by repetition)."""
    q, k, v = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    G = q.shape[1] // k.shape[1]
    k = torch.repeat_interleave(k, G, dim=1)
    v = torch.repeat_interleave(v, G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal,
                                                            scale=scale).numpy()


def pin_prefill_r_zero_is_sdpa(orc):
    q, r, k, v = rand_prefill(20, B=2, Hq=6, Hkv=3, L=17, D=8)
    for causal in (True, False):
        got = orc.parallax_prefill(q, np.zeros_like(r), k, v, 0.4, causal)
        close(got, torch_sdpa(q, k, v, 0.4, causal), 1e-12, f"prefill r=0 causal={causal}")


def pin_prefill_first_row_and_causality(orc):
    q, r, k, v = rand_prefill(21)
    o = orc.parallax_prefill(q, r, k, v, 0.3)
    close(o[:, :, 0], np.repeat(v[:, :, 0], 2, axis=1), 1e-12, "prefill row 0 = v_0")
    # rows 0..5 must not depend on keys or values at positions 6..L-1
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 6:] += 5.0 * np.random.default_rng(22).standard_normal(k2[:, :, 6:].shape)
    v2[:, :, 6:] = np.nan
    o2 = orc.parallax_prefill(q, r, k2, v2, 0.3)
    close(o2[:, :, :6], o[:, :, :6], 1e-12, "prefill causality")


def pin_prefill_local_linear_intercept(orc):
    """Causal row i with r_i = Sigma_w^{-1}(q_i - kbar) is the WLS intercept
    over keys 0..i (numpy lstsq), like the decode pin."""
    rng = np.random.default_rng(23)
    L, D, scale, i = 15, 4, 0.7, 13
    q = rng.standard_normal((1, 1, L, D))
    k = rng.standard_normal((1, 1, L, D))
    v = rng.standard_normal((1, 1, L, D))
    kk, vv, qi = k[0, 0, :i + 1], v[0, 0, :i + 1], q[0, 0, i]
    t = scale * kk @ qi
    w = np.exp(t - t.max())
    w /= w.sum()
    kbar = w @ kk
    sigma = (kk - kbar).T @ ((kk - kbar) * w[:, None])
    r = np.zeros_like(q)
    r[0, 0, i] = np.linalg.solve(sigma, qi - kbar)
    X = np.hstack([np.ones((i + 1, 1)), kk - qi])
    sw = np.sqrt(w)[:, None]
    coef, *_ = np.linalg.lstsq(X * sw, vv * sw, rcond=None)
    close(orc.parallax_prefill(q, r, k, v, scale)[0, 0, i], coef[0], 1e-9, "prefill LLA intercept")


def pin_prefill_gqa_mapping(orc):
    q, r, k, v = rand_prefill(24, Hq=8, Hkv=2)
    v[:, 0] = 1.0
    v[:, 1] = 2.0
    o = orc.parallax_prefill(q, r, k, v, 0.3)
    want = np.zeros_like(o)
    want[:, :4] = 1.0
    want[:, 4:] = 2.0
    close(o, want, 1e-12, "prefill GQA mapping")


# ------------------------------------------------------------------- varlen --

def rand_packed(seed, lens=(5, 0, 9, 1, 7), Hq=4, Hkv=2, D=8, r_scale=0.5):
    rng = np.random.default_rng(seed)
    total = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = rng.standard_normal((total, Hq, D))
    r = rng.standard_normal((total, Hq, D)) * r_scale
    k = rng.standard_normal((total, Hkv, D))
    v = rng.standard_normal((total, Hkv, D))
    return q, r, k, v, cu


def pin_varlen_r_zero_is_masked_sdpa(orc):
    """r = 0: torch's SDPA over the whole packed token axis with an explicit
    block-diagonal (and causal) boolean mask, computed independently of the
    per-sequence split."""
    q, r, k, v, cu = rand_packed(30)
    total = q.shape[0]
    seg = np.repeat(np.arange(len(cu) - 1), np.diff(cu))
    pos = np.arange(total)
    for causal in (True, False):
        mask = seg[:, None] == seg[None, :]
        if causal:
            mask &= pos[None, :] <= pos[:, None]
        qt, kt, vt = (torch.from_numpy(x.transpose(1, 0, 2).copy()) for x in (q, k, v))
        kt = torch.repeat_interleave(kt, 2, dim=0)
        vt = torch.repeat_interleave(vt, 2, dim=0)
        want = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=0.4).numpy().transpose(1, 0, 2)
        got = orc.parallax_varlen_prefill(q, np.zeros_like(r), k, v, cu, 0.4, causal)
        close(got, want, 1e-12, f"varlen r=0 causal={causal}")


def pin_varlen_equal_lengths_match_dense(orc):
    """Equal-length sequences packed along the token axis give the dense
    [B, H, L, D] forward, row for row."""
    q, r, k, v = rand_prefill(31, B=3, Hq=4, Hkv=2, L=6, D=8)
    dense = orc.parallax_prefill(q, r, k, v, 0.3)
    pack = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(-1, x.shape[1], x.shape[3]))
    cu = np.array([0, 6, 12, 18], dtype=np.int32)
    got = orc.parallax_varlen_prefill(pack(q), pack(r), pack(k), pack(v), cu, 0.3)
    close(got, pack(dense), 1e-12, "varlen = dense for equal lengths")


def pin_varlen_sequences_isolated(orc):
    """No row sees another sequence: replacing every token of one sequence
    (values by NaN) leaves the others' outputs bit-identical."""
    q, r, k, v, cu = rand_packed(32)
    o = orc.parallax_varlen_prefill(q, r, k, v, cu, 0.3)
    a, e = int(cu[2]), int(cu[3])  # the third sequence (9 tokens)
    q2, r2, k2, v2 = (x.copy() for x in (q, r, k, v))
    for x in (q2, r2, k2):
        x[a:e] += 3.0
    v2[a:e] = np.nan
    o2 = orc.parallax_varlen_prefill(q2, r2, k2, v2, cu, 0.3)
    keep = np.ones(q.shape[0], bool)
    keep[a:e] = False
    assert np.array_equal(o2[keep], o[keep]), "varlen sequences interact"
    # row 0 of every non-empty sequence is its own v_0
    for b in range(len(cu) - 1):
        if cu[b + 1] > cu[b]:
            close(o[cu[b]], np.repeat(v[cu[b]], 2, axis=0), 1e-12, "varlen first row")


# ------------------------------------------------------ paged, block-sparse --

def pin_paged_is_the_gathered_cache(orc):
    """Pages cut from a dense cache and scattered through the pool under a
    random table give the dense decode; with r = 0, torch's softmax attention."""
    q, r, k, v, n = rand_case(40, B=2, Hq=4, Hkv=2, D=8, Lmax=24, lengths=(11, 24))
    ps = 8  # small pages for the oracle (the kernel takes multiples of 64)
    pages = k.shape[2] // ps
    perm = np.random.default_rng(41).permutation(2 * pages)
    table = perm.reshape(2, pages).astype(np.int32)
    kp = np.zeros((2 * pages, ps, 2, 8))
    vp = np.zeros_like(kp)
    for b in range(2):
        for j in range(pages):
            kp[table[b, j]] = k[b, :, j * ps:(j + 1) * ps].transpose(1, 0, 2)
            vp[table[b, j]] = v[b, :, j * ps:(j + 1) * ps].transpose(1, 0, 2)
    got = orc.parallax_decode_paged(q, r, kp, vp, table, n, 0.3)
    close(got, orc.parallax_decode(q, r, k, v, n, 0.3), 1e-12, "paged = dense")
    got0 = orc.parallax_decode_paged(q, None, kp, vp, table, n, 0.3, probe=False)
    close(got0, torch_softmax_attention(q, k, v, n, 0.3), 1e-12, "paged r=0 = softmax")


def pin_block_sparse_selects_keys(orc):
    """r = 0 over a block list is softmax attention restricted to those keys
    (a boolean mask on torch's SDPA); all blocks listed is the dense decode; an
    empty list is a zero output."""
    rng = np.random.default_rng(42)
    B, Hq, Hkv, D, Lmax = 2, 4, 2, 8, 256
    q = rng.standard_normal((B, Hq, D))
    r = rng.standard_normal((B, Hq, D)) * 0.5
    k = rng.standard_normal((B, Hkv, Lmax, D))
    v = rng.standard_normal((B, Hkv, Lmax, D))
    n = np.array([200, 256], dtype=np.int32)
    ids = np.array([[0, 3, 2, 0], [1, 3, 0, 0]], dtype=np.int32)
    cnt = np.array([3, 2], dtype=np.int32)
    mask = np.zeros((B, Lmax), bool)
    for b in range(B):
        for blk in ids[b, :cnt[b]]:
            mask[b, 64 * blk:64 * blk + 64] = True
    mask &= np.arange(Lmax)[None] < n[:, None]
    qt = torch.from_numpy(q)[:, :, None]                      # [B, Hq, 1, D]
    kt = torch.repeat_interleave(torch.from_numpy(k), 2, dim=1)
    vt = torch.repeat_interleave(torch.from_numpy(v), 2, dim=1)
    want = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask)[:, None, None], scale=0.3)[:, :, 0].numpy()
    got = orc.parallax_decode_block_sparse(q, None, k, v, ids, cnt, n, 0.3, probe=False)
    close(got, want, 1e-12, "block-sparse r=0 = masked softmax")
    full = np.tile(np.arange(4, dtype=np.int32), (B, 1))
    close(orc.parallax_decode_block_sparse(q, r, k, v, full, np.array([4, 4]), n, 0.3),
          orc.parallax_decode(q, r, k, v, n, 0.3), 1e-12, "all blocks = dense")
    empty = orc.parallax_decode_block_sparse(q, r, k, v, ids, np.array([0, 2]), n, 0.3)
    assert np.all(empty[0] == 0.0) and np.all(np.isfinite(empty[1])), "empty block list"


PINS = [pin_hand_examples, pin_r_zero_is_softmax, pin_single_key_returns_v,
        pin_constant_values, pin_value_shift_and_scale, pin_key_translation,
        pin_linear_in_r, pin_key_permutation, pin_forms_agree,
        pin_local_linear_intercept, pin_gqa_mapping, pin_lengths_exact,
        pin_empty_sequence_is_zero, pin_prefill_r_zero_is_sdpa,
        pin_prefill_first_row_and_causality, pin_prefill_local_linear_intercept,
        pin_prefill_gqa_mapping, pin_varlen_r_zero_is_masked_sdpa,
        pin_varlen_equal_lengths_match_dense, pin_varlen_sequences_isolated,
        pin_paged_is_the_gathered_cache, pin_block_sparse_selects_keys]
