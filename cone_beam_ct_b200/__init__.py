"""B200-native cone-beam DRR ray-marcher (forward projection and its adjoint)."""
