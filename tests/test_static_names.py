"""Static check of the Python sources: every global name a function loads is
defined in its module or is a builtin, and every attribute taken on the
binding module (`sp.`) exists.  It catches a helper renamed or removed in one
place and still used in another -- in GPU tests too, which do not run here."""
import builtins
import dis
import glob
import importlib
import os
import re
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MODULES = (["bench", "__graft_entry__", "block_sparse_attention_33_b200",
            "block_sparse_attention_33_b200.sharding", "oracle.spattn_ref",
            "oracle.probe_residual", "oracle.hilbert", "workloads"]
           + ["tests." + os.path.basename(f)[:-3] for f in glob.glob(os.path.join(ROOT, "tests", "*.py"))])


def _code_objects(co):
    yield co
    for c in co.co_consts:
        if isinstance(c, types.CodeType):
            yield from _code_objects(c)


def test_no_undefined_globals():
    sys.path.insert(0, ROOT)
    bad = []
    for name in MODULES:
        mod = importlib.import_module(name)
        top = compile(open(mod.__file__).read(), mod.__file__, "exec")
        for co in _code_objects(top):
            if co is top:
                continue   # module level: names bound under `if __name__ == "__main__"` are fine
            for ins in dis.get_instructions(co):
                if ins.opname == "LOAD_GLOBAL" and not hasattr(mod, ins.argval) \
                        and not hasattr(builtins, ins.argval):
                    bad.append((name, co.co_name, ins.argval))
    assert not bad, bad


def test_binding_attributes_used_exist():
    sys.path.insert(0, ROOT)
    import block_sparse_attention_33_b200 as sp
    used = set()
    for f in glob.glob(os.path.join(ROOT, "tests", "*.py")) + [os.path.join(ROOT, "bench.py"),
                                                               os.path.join(ROOT, "__graft_entry__.py")]:
        used |= set(re.findall(r"\bsp\.([A-Za-z_]\w*)", open(f).read()))
    assert used and not [u for u in sorted(used) if not hasattr(sp, u)]
