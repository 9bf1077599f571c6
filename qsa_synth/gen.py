"""Counter-based generator (SplitMix64) and the value recipes built on it.

SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014; the 64-bit finaliser constants are Vigna's published
ones): the state advances by the golden-ratio increment and each output is the
state passed through a two-multiply xorshift finaliser.  Output number ``i`` of a
stream seeded with ``key`` is therefore ``mix(key + (i + 1) * GAMMA)``, which is
what makes every value addressable by its coordinates.

Value recipes (identical, bit for bit, in ``gen_cuda.cu``):

* integers uniform on [lo, hi]: Lemire's multiply-shift on the high 32 bits;
* "unit normal" bf16: Irwin-Hall sum of four 16-bit uniforms, centred and
  scaled to unit variance in fp64, rounded to fp32 (IEEE nearest) and then to
  bf16 (nearest, ties to even).  Every step is exactly specified, so the host
  and the device produce the same bits without sharing any code path.
"""

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_SQRT3 = 1.7320508075688772  # nearest fp64 to sqrt(3)

# tensor ids: one independent stream per input tensor
T_Q, T_K, T_V, T_IDXK, T_QIDX, T_W = 1, 2, 3, 4, 5, 6

_CHUNK = 1 << 22


def _u64(x):
    return np.asarray(x, dtype=np.uint64)


def _mix(z):
    z = _u64(z)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed, tensor_id):
    """Seed of the SplitMix64 stream for one tensor of one workload."""
    with np.errstate(over="ignore"):
        s = (_u64(seed) << np.uint64(32)) | _u64(tensor_id)
    return _mix(s)


def splitmix64_at(seed, tensor_id, idx):
    """Output number ``idx`` (uint64 array) of the tensor's SplitMix64 stream."""
    key = stream_key(seed, tensor_id)
    with np.errstate(over="ignore"):
        return _mix(key + (_u64(idx) + np.uint64(1)) * GAMMA)


def uniform_int(r, lo, hi):
    """Integers uniform on [lo, hi] from raw 64-bit draws (multiply-shift)."""
    n = np.uint64(hi - lo + 1)
    with np.errstate(over="ignore"):
        v = ((r >> np.uint64(32)) * n) >> np.uint64(32)
    return v.astype(np.int64) + lo


def _f32_to_bf16_bits(f):
    b = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def unit_normal_bf16_bits(r):
    """Approximately N(0,1) values as bf16 bit patterns (see module docstring)."""
    r = _u64(r)
    m = np.uint64(0xFFFF)
    s = ((r & m) + ((r >> np.uint64(16)) & m) + ((r >> np.uint64(32)) & m)
         + ((r >> np.uint64(48)) & m)).astype(np.float64)
    x = ((s + 2.0) / 65536.0 - 2.0) * _SQRT3
    return _f32_to_bf16_bits(x.astype(np.float32))


def int_to_bf16_bits(v):
    """Small integers (|v| < 256) are exact in bf16: plain truncation of fp32."""
    f = np.asarray(v, dtype=np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b):
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---- logical coordinates (independent of storage layout and capacity) ----

def q_coords(i, h, d):
    return (_u64(i) << np.uint64(16)) | (_u64(h) << np.uint64(8)) | _u64(d)


def qidx_coords(i, h, d):
    return q_coords(i, h, d)


def w_coords(i, h):
    return (_u64(i) << np.uint64(8)) | _u64(h)


def kv_coords(s, g, t, d):
    return ((((_u64(s) << np.uint64(8)) | _u64(g)) << np.uint64(32) | _u64(t)) << np.uint64(8)) | _u64(d)


def idxk_coords(s, t, d):
    return (((_u64(s) << np.uint64(32)) | _u64(t)) << np.uint64(8)) | _u64(d)


# ---- tensor generators (host) ----

def _chunked(coords_fn, shape, value_fn):
    out = np.empty(int(np.prod(shape)), dtype=np.uint16)
    flat = np.arange(out.size, dtype=np.int64)
    for c0 in range(0, out.size, _CHUNK):
        idx = np.unravel_index(flat[c0:c0 + _CHUNK], shape)
        out[c0:c0 + _CHUNK] = value_fn(coords_fn(*idx))
    return out.reshape(shape)


def gen_q(seed, query_ids, n_heads, head_dim):
    """Main-attention queries: bf16 bits [len(query_ids)][n_heads][head_dim]."""
    qid = np.asarray(query_ids, dtype=np.int64)
    shape = (qid.size, n_heads, head_dim)
    return _chunked(lambda a, h, d: q_coords(qid[a], h, d), shape,
                    lambda c: unit_normal_bf16_bits(splitmix64_at(seed, T_Q, c)))


def gen_kv_rows(seed, which, seq, tokens, n_kv_heads, head_dim):
    """K (which='k') or V (which='v') rows for the given tokens of one sequence.

    Returns bf16 bits [len(tokens)][n_kv_heads][head_dim]."""
    tid = T_K if which == "k" else T_V
    tok = np.asarray(tokens, dtype=np.int64)
    shape = (tok.size, n_kv_heads, head_dim)
    return _chunked(lambda a, g, d: kv_coords(seq, g, tok[a], d), shape,
                    lambda c: unit_normal_bf16_bits(splitmix64_at(seed, tid, c)))


def gen_idx_k(seed, seq, t0, t1, idx_dim, lo=-4, hi=4):
    """Per-token indexer keys, integers uniform on [lo, hi] as bf16 bits [t1-t0][idx_dim]."""
    shape = (t1 - t0, idx_dim)
    return _chunked(lambda a, d: idxk_coords(seq, a + t0, d), shape,
                    lambda c: int_to_bf16_bits(uniform_int(splitmix64_at(seed, T_IDXK, c), lo, hi)))


def gen_q_idx(seed, query_ids, n_idx_heads, idx_dim, lo=-4, hi=4):
    """Indexer queries, integers uniform on [lo, hi] as bf16 bits [n][n_idx_heads][idx_dim]."""
    qid = np.asarray(query_ids, dtype=np.int64)
    shape = (qid.size, n_idx_heads, idx_dim)
    return _chunked(lambda a, h, d: qidx_coords(qid[a], h, d), shape,
                    lambda c: int_to_bf16_bits(uniform_int(splitmix64_at(seed, T_QIDX, c), lo, hi)))


def gen_w(seed, query_ids, n_idx_heads, lo=1, hi=3):
    """Indexer head weights, integers uniform on [lo, hi] as float32 [n][n_idx_heads]."""
    qid = np.asarray(query_ids, dtype=np.int64)
    a, h = np.meshgrid(qid, np.arange(n_idx_heads), indexing="ij")
    v = uniform_int(splitmix64_at(seed, T_W, w_coords(a, h)), lo, hi)
    return v.astype(np.float32)
