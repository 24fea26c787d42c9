"""Pytest plugin used by ``test_oracle_mutations``: when ORACLE_MUTATION is
set it plants one mistake in the oracle before any test module imports it.

The variable holds JSON [module, qualified function name, old text, new
text].  The function's source must contain the old text exactly once; the
edited source is compiled in the module's globals and its code object
replaces the original function's, so every reference to the function (the
names test modules imported) runs the mistake.  Only ever used on the CPU
oracle, in a child process."""
import importlib
import inspect
import json
import os
import textwrap


def _plant(spec):
    mod_name, qualname, old, new = spec
    mod = importlib.import_module(mod_name)
    fn = mod
    for part in qualname.split("."):
        fn = getattr(fn, part)
    src = textwrap.dedent(inspect.getsource(fn))
    if src.count(old) != 1:
        raise RuntimeError(f"mutation site not unique in {qualname}: {old!r}")
    ns = {}
    exec(compile(src.replace(old, new), mod.__file__, "exec"), mod.__dict__, ns)
    fn.__code__ = ns[qualname.split(".")[-1]].__code__


_spec = os.environ.get("ORACLE_MUTATION")
if _spec:
    _plant(json.loads(_spec))
