"""The C ABI library on the host: it loads, exports every declared entry
point, and rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("moe_b200.h", "gdn_b200.h")]


def declared_functions():
    names = set()
    for header in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(header).read(), flags=re.S)
        names |= set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b((?:moe|gdn)_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


def test_header_declares_the_layer_calls():
    names = declared_functions()
    for n in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_workspace_size",
              "moe_get_device_error", "moe_gather_rows", "gdn_scan", "moe_router_logits"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import bit_dequant_expert_b200 as m
    lib = ctypes.CDLL(m.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(declared_functions()) <= set(m.EXPORTED) | {"moe_status_string"}


def test_workspace_size_and_config_checks():
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    n1, n2 = m.moe_workspace_size(cfg, 1), m.moe_workspace_size(cfg, 2048)
    assert 0 < n1 < n2 and n1 % 256 == 0 and n2 % 256 == 0
    # (k+1) T I bf16 rows of h, T E fp32 logits at least
    assert n2 >= 9 * 2048 * 512 * 2 + 2048 * 256 * 4
    for bad in (m.config(hidden=300), m.config(inter=100), m.config(num_experts=0), m.config(num_experts=257),
                m.config(top_k=0), m.config(top_k=9), m.config(num_experts=4, top_k=8),
                m.config(group_size=32), m.config(has_shared=2)):
        assert m.moe_workspace_size(bad, 16) == 0
    # an expert-parallel shard: fewer experts, one pair per row
    assert m.moe_workspace_size(m.config(num_experts=128, top_k=1, has_shared=0), 4096) > 0
    assert m.moe_workspace_size(m.config(num_experts=32, top_k=4), 16) > 0
    assert m.moe_workspace_size(cfg, 0) == 0
    assert m.moe_workspace_size(cfg, 65537) == 0


FAKE = 0x7F0000000000   # 256-byte aligned, never dereferenced: every case fails validation first


def _route(cfg, T, ws_bytes, ws=FAKE, idx=FAKE, x=FAKE):
    import bit_dequant_expert_b200 as m
    return m.moe_route(cfg, T, x, FAKE, None, None, 0, idx, FAKE, FAKE, ws, ws_bytes=ws_bytes, stream=0,
                       raise_on_error=False)


def test_host_validation_before_launch():
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    need = m.moe_workspace_size(cfg, 64)
    assert _route(cfg, 0, need) == m.MOE_ERR_INVALID_ARG
    assert _route(m.config(hidden=1000), 64, need) == m.MOE_ERR_UNSUPPORTED
    assert _route(cfg, 64, need - 256) == m.MOE_ERR_WORKSPACE
    assert _route(cfg, 64, need, ws=FAKE + 16) == m.MOE_ERR_WORKSPACE
    assert _route(cfg, 64, need, ws=None) == m.MOE_ERR_WORKSPACE
    assert _route(cfg, 64, need, idx=None) == m.MOE_ERR_INVALID_ARG
    assert _route(cfg, 64, need, x=FAKE + 2) == m.MOE_ERR_INVALID_ARG
    st = m.moe_permute(cfg, 64, FAKE, None, None, FAKE, FAKE, FAKE, ws_bytes=need, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_INVALID_ARG
    st = m.moe_expert_ffn(cfg, 64, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 7, FAKE, FAKE, FAKE,
                          ws_bytes=need, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_INVALID_ARG
    st = m.moe_expert_ffn(cfg, 64, FAKE, FAKE + 16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, None, FAKE,
                          ws_bytes=need, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_INVALID_ARG      # packed weights must be 256-byte aligned
    st = m.moe_expert_ffn_path(cfg, 64, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, FAKE, None, FAKE, 0,
                               ws_bytes=need, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_INVALID_ARG      # pairs mode with a shared expert needs out1
    st = m.moe_combine(cfg, 64, 1, FAKE, FAKE, None, FAKE, FAKE, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_INVALID_ARG
    def logits(T=64, x=FAKE, out=FAKE, bias=None, stride=0, ws=FAKE, c=cfg):
        return m.moe_router_logits(c, T, x, FAKE, bias, stride, out, ws, ws_bytes=need, stream=0,
                                   raise_on_error=False)

    assert logits(T=0) == m.MOE_ERR_INVALID_ARG
    assert logits(x=None) == m.MOE_ERR_INVALID_ARG
    assert logits(x=FAKE + 8) == m.MOE_ERR_INVALID_ARG
    assert logits(out=FAKE + 4) == m.MOE_ERR_INVALID_ARG
    assert logits(bias=FAKE + 2) == m.MOE_ERR_INVALID_ARG
    assert logits(bias=FAKE, stride=-1) == m.MOE_ERR_INVALID_ARG
    assert logits(ws=None) == m.MOE_ERR_WORKSPACE
    assert logits(c=m.config(num_experts=128, top_k=1, has_shared=0)) == m.MOE_ERR_UNSUPPORTED
    assert m.moe_get_device_error(None, 0) == m.MOE_ERR_WORKSPACE
    assert m.moe_status_string(m.MOE_ERR_NONFINITE) == "MOE_ERR_NONFINITE"


def test_expert_shard_validation_before_launch():
    """An expert shard (fewer experts, top_k 1) may run the expert FFN, the
    row gather and the scatter combine; the router, the permutation, the pairs
    combine and the fused decode layer stay at 256 experts, top 8."""
    import bit_dequant_expert_b200 as m
    sh = m.config(num_experts=128, top_k=1, has_shared=0)
    need = m.moe_workspace_size(sh, 64)
    assert _route(sh, 64, need) == m.MOE_ERR_UNSUPPORTED
    st = m.moe_permute(sh, 64, FAKE, None, FAKE, FAKE, FAKE, FAKE, ws_bytes=need, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_UNSUPPORTED
    assert _decode(m.config(num_experts=128), 1, m.moe_workspace_size(m.config(num_experts=128), 1)) == \
        m.MOE_ERR_UNSUPPORTED
    st = m.moe_combine(sh, 64, m.MOE_MODE_PAIRS, FAKE, None, FAKE, FAKE, FAKE, stream=0, raise_on_error=False)
    assert st == m.MOE_ERR_UNSUPPORTED
    # the row gather: the block must lie inside [0, T*k), the pointers be set and aligned
    cfg = m.config()
    full = m.moe_workspace_size(cfg, 64)

    def gather(T=64, begin=0, n=8, x=FAKE, rows=FAKE, w=None, ws=FAKE, nbytes=full):
        return m.moe_gather_rows(cfg, T, x, FAKE, None, begin, n, rows, w, ws, ws_bytes=nbytes, stream=0,
                                 raise_on_error=False)

    assert gather(begin=-1) == m.MOE_ERR_INVALID_ARG
    assert gather(begin=500, n=13) == m.MOE_ERR_INVALID_ARG
    assert gather(n=-1) == m.MOE_ERR_INVALID_ARG
    assert gather(n=0, x=None, rows=None) == m.MOE_OK       # nothing to copy, nothing launched
    assert gather(x=None) == m.MOE_ERR_INVALID_ARG
    assert gather(rows=FAKE + 8) == m.MOE_ERR_INVALID_ARG
    assert gather(w=FAKE + 2) == m.MOE_ERR_INVALID_ARG
    assert gather(ws=None) == m.MOE_ERR_WORKSPACE
    assert gather(nbytes=256) == m.MOE_ERR_WORKSPACE


def _decode(cfg, T, ws_bytes, x=FAKE, y=FAKE, bias=None, stride=0):
    import bit_dequant_expert_b200 as m
    return m.moe_decode_layer(cfg, T, x, FAKE, bias, stride, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              FAKE, FAKE, y, FAKE, ws_bytes=ws_bytes, stream=0, raise_on_error=False)


def test_decode_layer_validation_before_launch():
    """The fused decode call takes 1 <= T <= 8 at hidden 512/1024/2048; anything
    else, a bad pointer or a short workspace is refused before any launch."""
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    need = m.moe_workspace_size(cfg, 16)
    assert _decode(cfg, 9, need) == m.MOE_ERR_UNSUPPORTED
    assert _decode(m.config(hidden=4096), 1, m.moe_workspace_size(m.config(hidden=4096), 1)) == m.MOE_ERR_UNSUPPORTED
    assert _decode(cfg, 0, need) == m.MOE_ERR_INVALID_ARG
    assert _decode(cfg, 8, 256) == m.MOE_ERR_WORKSPACE
    assert _decode(cfg, 8, need, x=None) == m.MOE_ERR_INVALID_ARG
    assert _decode(cfg, 8, need, y=FAKE + 8) == m.MOE_ERR_INVALID_ARG
    assert _decode(cfg, 8, need, bias=FAKE, stride=-1) == m.MOE_ERR_INVALID_ARG


def test_wait_selftest_validation_before_launch():
    """The failure-detection self-test refuses a bad kind, CTA count,
    suppressed CTA, wait limit or workspace before launching anything."""
    import bit_dequant_expert_b200 as m

    def call(kind=1, ctas=4, skip=1, limit=1_000_000, ws=FAKE):
        return m.moe_wait_selftest(kind, ctas, skip, limit, ws, stream=0, raise_on_error=False)

    assert call(ws=None) == m.MOE_ERR_WORKSPACE
    assert call(ws=FAKE + 16) == m.MOE_ERR_WORKSPACE
    assert call(kind=2) == m.MOE_ERR_INVALID_ARG
    assert call(kind=-1) == m.MOE_ERR_INVALID_ARG
    assert call(kind=0, ctas=2, skip=-1) == m.MOE_ERR_INVALID_ARG
    assert call(kind=0, ctas=1, skip=0) == m.MOE_ERR_INVALID_ARG
    assert call(ctas=0, skip=-1) == m.MOE_ERR_INVALID_ARG
    assert call(ctas=149, skip=-1) == m.MOE_ERR_INVALID_ARG
    assert call(ctas=4, skip=4) == m.MOE_ERR_INVALID_ARG
    assert call(ctas=4, skip=-2) == m.MOE_ERR_INVALID_ARG
    assert call(limit=999) == m.MOE_ERR_INVALID_ARG
    assert call(limit=1_000_000_001) == m.MOE_ERR_INVALID_ARG


def test_launch_count_per_path():
    """Kernels per layer as the bench counts them (host-only, no device needed)."""
    import bit_dequant_expert_b200 as m
    cfg = m.config()
    SC, PA = m.MOE_MODE_SCATTER, m.MOE_MODE_PAIRS
    # route (small T: one launch) + permute (T <= 256: one) + decode FFN (one) + combine
    assert m.moe_launch_count(cfg, 1, SC, m.MOE_PATH_AUTO) == 4
    # the decode kernel only accumulates y_acc: bf16 rows go to the tensor-core path (gather + 2)
    assert m.moe_launch_count(cfg, 1, PA, m.MOE_PATH_AUTO) == 1 + 1 + 3 + 1
    # T = 2048: router logits + top-k, three permute kernels, gather + two GEMMs, combine
    assert m.moe_launch_count(cfg, 2048, PA, m.MOE_PATH_AUTO) == 2 + 3 + 3 + 1
    assert m.moe_launch_count(cfg, 2048, SC, m.MOE_PATH_SIMT) == 2 + 3 + 2 + 1
    assert m.moe_launch_count(cfg, 2048, SC, m.MOE_PATH_GEMV) == -1      # more than 8 tokens
    assert m.moe_launch_count(cfg, 4, 7, m.MOE_PATH_AUTO) == -1          # no such mode
    assert m.moe_launch_count(cfg, 0, SC, m.MOE_PATH_AUTO) == -1


def test_gdn_scan_validation_before_launch():
    """The scan refuses counts below 1, null or misaligned pointers and head
    sizes other than 128 before launching anything."""
    import bit_dequant_expert_b200 as m

    def call(B=1, T=4, Hk=2, Hv=4, dk=128, dv=128, q=FAKE, g=FAKE, s_out=FAKE, o=FAKE):
        return m.gdn_scan(B, T, Hk, Hv, dk, dv, q, FAKE, FAKE, g, FAKE, 0.1, FAKE, s_out, o, stream=0,
                          raise_on_error=False)

    assert call(B=0) == m.MOE_ERR_INVALID_ARG
    assert call(T=0) == m.MOE_ERR_INVALID_ARG
    assert call(q=None) == m.MOE_ERR_INVALID_ARG
    assert call(q=FAKE + 8) == m.MOE_ERR_INVALID_ARG
    assert call(o=FAKE + 2) == m.MOE_ERR_INVALID_ARG
    assert call(g=FAKE + 2) == m.MOE_ERR_INVALID_ARG
    assert call(s_out=None) == m.MOE_ERR_INVALID_ARG
    assert call(dk=64) == m.MOE_ERR_UNSUPPORTED
    assert call(dv=256) == m.MOE_ERR_UNSUPPORTED
    assert call(Hk=3, Hv=4) == m.MOE_ERR_UNSUPPORTED
