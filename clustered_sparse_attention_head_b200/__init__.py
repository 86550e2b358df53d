"""AdaCluster clustered sparse attention on B200 (sm_100a).

The compute path is libadacluster.so (include/adacluster.h); ``api.AdaCluster``
is its Python front end.  ``workloads`` draws the seeded synthetic inputs.
"""
from . import workloads  # noqa: F401


def build(force: bool = False) -> str:
    from ._build import build as _b
    return _b(force=force)


def AdaCluster(*a, **k):  # noqa: N802 - thin alias that imports torch lazily
    from .api import AdaCluster as _A
    return _A(*a, **k)


def Config(*a, **k):  # noqa: N802
    from .api import Config as _C
    return _C(*a, **k)
