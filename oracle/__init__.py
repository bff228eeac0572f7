"""CPU oracle for the ConvRot linear (test infrastructure, see convrot_ref)."""
from . import convrot_ref  # noqa: F401
