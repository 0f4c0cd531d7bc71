#pragma once
// The decoder kernels need nothing from the encoder's device header.
