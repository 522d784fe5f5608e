"""One routed-MoE layer, restated plainly in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Method (FreeToken linux, "FreeToken's MoE memory handling"): per token the
router scores every routed expert, a few experts are activated, each active
expert's FFN runs on the token, and the outputs are mixed by the gate weights.
Caching decides only where expert weights are read from, so the result equals
the plain dense definition (FreeToken RTX 5090, dynamic reconfiguration:
capacity affects performance, not correctness).
"""
import numpy as np

# ----------------------------------------------------------------- formats --


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact): a bf16 is the top half of a float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_int4(packed: np.ndarray) -> np.ndarray:
    """Packed nibbles [R, K/2] -> int values [R, K] in [-8, 7].

    READING (the pages name a 4-bit release but no layout): byte b of a row holds
    element 2b in its low nibble and element 2b+1 in its high nibble, each a
    4-bit two's-complement integer: codes 0..7 stand for themselves, codes 8..15
    for code - 16.
    """
    p = np.asarray(packed, dtype=np.uint8)
    code = np.arange(16, dtype=np.int64)
    value_of_code = np.where(code >= 8, code - 16, code)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int64)
    out[:, 0::2] = value_of_code[p & 0x0F]
    out[:, 1::2] = value_of_code[p >> 4]
    return out


def dequant_int4(packed: np.ndarray, scale_bits: np.ndarray) -> np.ndarray:
    """w = q * s, s the bf16 scale of each group of 128 consecutive reduction-axis
    elements of a row (READING: symmetric int4, group 128 along K)."""
    q = decode_int4(packed).astype(np.float64)
    s = widen_bf16(scale_bits)
    R = q.shape[0]
    return (q.reshape(R, -1, 128) * s[:, :, None]).reshape(R, -1)


def decode_e2m1(codes: np.ndarray) -> np.ndarray:
    """FP4 E2M1 codes (0..15) -> float64.  Bit 3 sign, bits 2-1 exponent (bias 1), bit 0
    mantissa; exponent 0 is subnormal: m * 0.5.  (The OCP microscaling FP4 element.)"""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, m * 0.5, (1.0 + m * 0.5) * np.power(2.0, e - 1))
    return sign * mag


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """FP8 E4M3 codes -> float64.  Bit 7 sign, bits 6-3 exponent (bias 7), bits 2-0
    mantissa; exponent 0 is subnormal: m/8 * 2^-6; no infinities (0x7F/0xFF are NaN)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.power(2.0, e - 7))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def dequant_nvfp4(packed: np.ndarray, scale_codes: np.ndarray, g: float) -> np.ndarray:
    """w = e2m1(q) * e4m3(s) * g, s shared by 16 consecutive reduction-axis elements
    of a row (READING of the pages' NVFP4 release: the 16-element micro-block with an
    E4M3 scale and an FP32 tensor scale; element 2b in the low nibble of byte b)."""
    p = np.asarray(packed, dtype=np.uint8)
    codes = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int64)
    codes[:, 0::2] = p & 0x0F
    codes[:, 1::2] = p >> 4
    s = decode_e4m3(scale_codes)
    return decode_e2m1(codes) * np.repeat(s, 16, axis=1) * float(g)


def expert_weights(blob: np.ndarray, wdtype: str, H: int, I: int):
    """Decode one expert blob into (W_gate [I,H], W_up [I,H], W_down [H,I]) float64.

    Blob layout (the runtime layout of an expert bank; the pages' FTW format
    stores experts "in runtime layout" without giving it - FreeToken linux,
    setup, "prepare the model weights"): the three matrices row-major, gate,
    up, down; for int4, the three packed matrices and then their three scale
    arrays; for nvfp4, the three packed e2m1 matrices, their three e4m3 block-scale
    arrays and the three fp32 global scales.
    """
    blob = np.asarray(blob, dtype=np.uint8).reshape(-1)
    m = H * I
    if wdtype == "f32":
        w = blob.view(np.float32).astype(np.float64)
        return w[:m].reshape(I, H), w[m:2 * m].reshape(I, H), w[2 * m:3 * m].reshape(H, I)
    if wdtype == "bf16":
        w = widen_bf16(blob.view(np.uint16))
        return w[:m].reshape(I, H), w[m:2 * m].reshape(I, H), w[2 * m:3 * m].reshape(H, I)
    if wdtype == "nvfp4":
        q = blob[:3 * m // 2]
        s = blob[3 * m // 2:3 * m // 2 + 3 * m // 16]
        g = blob[3 * m // 2 + 3 * m // 16:3 * m // 2 + 3 * m // 16 + 12].view(np.float32).astype(np.float64)
        n = m // 16
        wg = dequant_nvfp4(q[:m // 2].reshape(I, H // 2), s[:n].reshape(I, H // 16), g[0])
        wu = dequant_nvfp4(q[m // 2:m].reshape(I, H // 2), s[n:2 * n].reshape(I, H // 16), g[1])
        wd = dequant_nvfp4(q[m:3 * m // 2].reshape(H, I // 2), s[2 * n:3 * n].reshape(H, I // 16), g[2])
        return wg, wu, wd
    if wdtype == "int4":
        q = blob[:3 * m // 2]
        s = blob[3 * m // 2:].view(np.uint16)
        g = m // 128
        wg = dequant_int4(q[:m // 2].reshape(I, H // 2), s[:g].reshape(I, H // 128))
        wu = dequant_int4(q[m // 2:m].reshape(I, H // 2), s[g:2 * g].reshape(I, H // 128))
        wd = dequant_int4(q[m:3 * m // 2].reshape(H, I // 2), s[2 * g:3 * g].reshape(H, I // 128))
        return wg, wu, wd
    raise ValueError(wdtype)


# ----------------------------------------------------------------- routing --


def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """z[t, e] = sum_h x[t, h] * W_r[e, h], formed in float64 and rounded once to float32.

    READING: the logits are float32 (the stated workloads fix fp32 router
    logits), so top-k below is decided on float32 values, as in the kernel.
    """
    z = np.asarray(x, dtype=np.float64) @ np.asarray(w_router, dtype=np.float64).T
    return z.astype(np.float32)


def topk(z: np.ndarray, k: int):
    """The k experts with the largest logit per token (FreeToken linux: the router
    activates only a few experts per token, e.g. 6 of 256).

    READING: ties go to the lower expert index; ids are listed by descending
    logit (equal logits: ascending index).  Also returns, per token, the gap
    z_(k) - z_(k+1) between the last selected and the first unselected logit
    (inf when k == E), so a caller can tell near-ties apart.
    """
    z = np.asarray(z, dtype=np.float32)
    T, E = z.shape
    ids = np.empty((T, k), dtype=np.int32)
    gap = np.full(T, np.inf)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(z[t, e]), e))
        ids[t] = order[:k]
        if k < E:
            gap[t] = float(z[t, order[k - 1]]) - float(z[t, order[k]])
    return ids, gap


def gates(z_sel: np.ndarray, gating: str) -> np.ndarray:
    """Gate weights over the k selected experts, normalised to sum to 1.

    softmax: g_j = exp(z_j) / sum_sel exp(z)  (the full softmax restricted to the
             selected experts and renormalised).
    sigmoid: g_j = sigma(z_j) / sum_sel sigma(z).
    The pages give neither formula (stated workloads).
    """
    zs = np.asarray(z_sel, dtype=np.float64)
    if gating == "softmax":
        e = np.exp(zs - zs.max(axis=1, keepdims=True))
    elif gating == "sigmoid":
        e = 1.0 / (1.0 + np.exp(-zs))
    else:
        raise ValueError(gating)
    return e / e.sum(axis=1, keepdims=True)


def selected_set(ids: np.ndarray) -> np.ndarray:
    """S: the sorted distinct experts chosen by any token of the batch - the experts
    whose weights one forward reads (FreeToken linux, "FreeToken's MoE memory
    handling": only the experts the router asks for are brought to the GPU)."""
    return np.unique(np.asarray(ids).reshape(-1)).astype(np.int32)


def permute(ids: np.ndarray, E: int):
    """Expert-major order of the (token, slot) pairs of a batch.

    counts[e] = number of pairs routed to e; offsets = exclusive prefix sum
    (length E+1); perm lists the flat pair index t*k + j grouped by expert in
    ascending expert order and, inside an expert, by ascending token.
    READING: the pages give no grouping; this stable order is the plainest one
    that lets each expert's weights be read once per forward.
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            counts[ids[t, j]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    perm = np.empty(T * k, dtype=np.int64)
    fill = offsets[:-1].copy()
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            perm[fill[e]] = t * k + j
            fill[e] += 1
    return counts, offsets, perm


# --------------------------------------------------------------- expert FFN --


def silu(a: np.ndarray) -> np.ndarray:
    """silu(a) = a * sigmoid(a).  READING: the pages name no expert FFN; the stated
    workloads use SwiGLU experts, whose activation this is."""
    return a / (1.0 + np.exp(-a))


def swiglu_ffn(a: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """y = W_down (silu(W_gate a) * (W_up a)) for each row a of `a` [n, H].

    READING: one routed expert is a SwiGLU FFN with gate and up [I, H] and down
    [H, I] (the stated workloads; the pages only say that each active expert runs
    on the token - FreeToken linux, "FreeToken's MoE memory handling")."""
    a = np.asarray(a, dtype=np.float64)
    u = a @ w_gate.T
    v = a @ w_up.T
    h = silu(u) * v
    return h @ w_down.T


# ---------------------------------------------------------------- one layer --


def route(x, w_router, k, gating):
    """Router + top-k + gates for a batch: returns dict(ids, gates, gap, z).
    (FreeToken linux, "FreeToken's MoE memory handling": the router picks a few
    experts per token; the readings are those of router_logits, topk and gates.)"""
    z = router_logits(x, w_router)
    ids, gap = topk(z, k)
    z_sel = np.take_along_axis(z, ids.astype(np.int64), axis=1)
    return {"ids": ids, "gates": gates(z_sel, gating), "gap": gap, "z": z}


def experts_and_combine(x, ids, g, E, wdtype, H, I, blob_of, shared_blob=None):
    """Permute the (token, slot) pairs by expert, run each selected expert's FFN on
    its tokens, and mix: out[t] = sum_{j<k} g[t,j] * y[t,j] (+ shared FFN(x_t)),
    the sum taken in ascending j.

    (FreeToken linux, "FreeToken's MoE memory handling": each active expert runs on
    the token and the outputs are mixed by the gate weights.  READINGS: the mixing
    order is ascending j; a shared expert is added with weight 1.)"""
    x = np.asarray(x, dtype=np.float64)
    T, k = ids.shape
    counts, offsets, perm = permute(ids, E)
    y = np.zeros((T * k, H))
    for e in range(E):
        if counts[e] == 0:
            continue
        pairs = perm[offsets[e]:offsets[e + 1]]
        tok = pairs // k
        wg, wu, wd = expert_weights(blob_of(e), wdtype, H, I)
        y[pairs] = swiglu_ffn(x[tok], wg, wu, wd)
    out = np.zeros((T, H))
    for j in range(k):
        out += g[:, j:j + 1] * y[np.arange(T) * k + j]
    if shared_blob is not None:
        wg, wu, wd = expert_weights(shared_blob, wdtype, H, I)
        out += swiglu_ffn(x, wg, wu, wd)
    return out


def moe_layer(x, w_router, k, gating, wdtype, H, I, blob_of, shared_blob=None):
    """One routed-MoE layer on a batch x [T, H].

    blob_of(e) returns the bytes of routed expert e (from wherever the caller
    keeps them: the host pool, or a cache slot).  shared_blob, if given, is the
    always-on shared expert, added with weight 1 (READING: the pages name no
    shared-expert weight).

    out[t] = sum_{j<k} g[t,j] * FFN_{ids[t,j]}(x_t)  (+ FFN_shared(x_t)),
    the sum taken in ascending j.  Returns dict(out, ids, gates, gap, z).
    """
    r = route(x, w_router, k, gating)
    out = experts_and_combine(x, r["ids"], r["gates"], w_router.shape[0], wdtype, H, I, blob_of,
                              shared_blob)
    return {"out": out, **r}
