from . import inputs  # noqa: F401
